// NF4 GEMV for small batches (M <= 16 tokens), HBM-bound:
//   Zc = bf16(c·X·A),   Y = X·Ŵ + Zc·B,   Ŵ decoded on the fly.
//
// Page "QLoRA：冻结的 4-bit 权重怎样参与一次微调", §量化基座与可训练支路怎样相加
// (Y = X·Ŵ + c·Z·B with Z = X·A), in the decode-like case where a few tokens
// stream the whole 0.5 byte per weight payload.
//
// Work split.  The weight's columns are cut into groups of 256 (four NF4
// blocks) and its K rows into S contiguous ranges of whole 128-row stages.
// The S CTAs of one column group form a thread-block cluster (1 x S x 1), one
// CTA per SM.  Each CTA streams its stages (packed 128 x 128 bytes, X 16 x 128
// bf16, and 128 rows of A, all by TMA) through a ring in shared memory.  At the
// end the cluster adds the S partial sums of every output in split order
// through distributed shared memory: no workspace, no second launch, and the
// bits do not depend on timing.
//
// Products.  y[m][n] = sum_k x[m][k] Ŵ[k][n] runs on mma.sync m16n8k16 with a
// 16-token tile and the block scale folded into the activation:
//   y[m][n] = sum_k bf16(x[m][k] * a'[k][n/64]) * bf16(C_code(k, n)),
// so the weight operand is the codebook value bf16(C_j) and needs no per-block
// table: a 256-entry table of bf16 pairs (C[hi nibble], C[lo nibble]) turns one
// byte into one fragment register.  That byte is built from two adjacent
// weight rows (k, k+1) at one column by interleaving nibbles of their packed
// words, so each lookup yields the (k, k+1) pair a fragment register holds.
// The table is held 32 times, one copy per bank ((byte << 8) | lane * 4
// addresses a lane's own copy), so lookups never conflict; it sits at the start
// of the dynamic shared window, so its base is a constant of the load.  Inside
// a 64-column block, n-tile f of the fragments' rows g covers weight columns
// 8g + 2f and 8g + 2f + 1, so lane group g reads one packed word per row.
// Against x · bf16(C·a'), every product carries at most one more bf16 rounding
// (of x·a'), relative 2^-9.
//
// X·A.  Each CTA also multiplies the raw activation fragments (the same
// registers) by its K range of A (staged rows of A read with ldmatrix.trans).
// The cluster adds these slices in split order like the outputs, so every
// cluster holds the same full X·A; each rounds Zc = bf16(c·X·A) once, adds Zc·B
// to its outputs, and the first cluster writes Zc.  Launched with one column
// group and `zc_only`, the kernel forms Zc alone with the same splits and the
// same sums: that is the backward's recompute of Zc, bit-identical to the
// forward's.
#include "common.cuh"
#include "kernels.cuh"
#include "profile.cuh"
#include "tmap.cuh"

namespace qnf4 {

namespace {

__constant__ float kCodeVals[32] = {QNF4_TABLE_VALUES, QNF4_INT4_VALUES};   // NF4, INT4

constexpr int kGvTable = 65536;          // 256 entries x 64 words (32 used) x 4 B
constexpr int kGvRows = 128;             // k rows per stage
constexpr int kGvCols = 256;             // weight columns per CTA (four NF4 blocks)
constexpr int kGvMaxStages = 6;
constexpr int kGvPk = kGvRows * 128;     // packed weights of a stage
constexpr int kGvXb = 2 * 2048;          // 16 tokens x 128 k bf16, two swizzled 64-k halves
constexpr int kGvCompute = 16;           // compute warps: 4 column blocks x 4 row slots
constexpr int kGvScaleWarps = 3;         // scale warps, taking stages in turn
constexpr int kGvWarps = kGvCompute + 1 + kGvScaleWarps;   // + the TMA producer
constexpr int kGvThreads = kGvWarps * 32;
constexpr int kGvScaleWords = 4 * kGvRows;   // decode scales of one stage: 4 blocks x 128 rows
constexpr int kGvSmemMax = 232448;       // 227 KB, the opt-in limit per CTA
constexpr int kGvPLd = kGvCols + 4;      // fp32 words per token row of a CTA's sums
// epilogue regions, carved from the ring once every stage is consumed
constexpr int kGvRedOff = 0;                         // [12 warps][32 regs][32 lanes] fp32
constexpr int kGvZredOff = kGvRedOff + 12 * 1024 * 4;  // [12 warps][8 regs][32 lanes] fp32
constexpr int kGvPsOff = kGvZredOff + 12 * 256 * 4;  // [16 tokens][kGvPLd] fp32, this CTA's sums
constexpr int kGvZsOff = kGvPsOff + 16 * kGvPLd * 4;  // [16][64] fp32, this CTA's X·A slice
constexpr int kGvZcOff = kGvZsOff + 16 * 64 * 4;     // [16][64] fp32, the rounded Zc
constexpr int kGvEpilogueBytes = kGvZcOff + 16 * 64 * 4;

struct GemvArgs {
  int M, K, N, r;
  int rp;               // rows of the staged B tile (r rounded up to a multiple of 8)
  int rp2;              // width of the staged rows of A (power of two >= 8, >= rp)
  int nstages;          // ring depth
  int stage_bytes;      // packed + X + A bytes of a stage (a multiple of 1024)
  int stages_per_split; // 128-row stages per CTA of a cluster
  int zc_only;          // 1: compute and write Zc only (no weights, no Y)
  float c;
  ScaleView sv;
  uint16_t* Y;          // M x N
  uint16_t* Zc;         // M x ldz, written by CTA (0, 0); columns r .. ldz-1 get 0
  int ldz;
  int32_t* d_status;
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lds32(uint32_t saddr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(saddr));
  return v;
}

__device__ __forceinline__ void ldsm_x2_trans(uint32_t saddr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(saddr));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Raw scale loads of one (row, block), issued stages ahead of their use.
struct GvScale {
  uint32_t q;   // code8 (double quantization)
  float v;      // s2 of the block's 256-group, or the fp32 absmax
};

__device__ __forceinline__ GvScale gemv_scale_load(const ScaleView& sv, int64_t b) {
  GvScale r;
  r.q = 0u;
  if (sv.code8 == nullptr) {
    asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(r.v) : "l"(sv.absmax + b));
  } else {
    uint16_t q;
    asm volatile("ld.global.nc.u8 %0, [%1];" : "=h"(q) : "l"(sv.code8 + b));
    asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(r.v) : "l"(sv.s2 + (b >> 8)));
    r.q = q;
  }
  return r;
}

// The value at `off` in the first S CTAs of the cluster, added in rank order
// (all loads in flight before the first add).
__device__ __forceinline__ float cluster_sum_in_order(uint32_t off, int S) {
  float part[8];
#pragma unroll
  for (int sp = 0; sp < 8; ++sp) part[sp] = sp < S ? ld_dsmem_f32(off, static_cast<uint32_t>(sp)) : 0.0f;
  float a = 0.0f;
#pragma unroll
  for (int sp = 0; sp < 8; ++sp)
    if (sp < S) a += part[sp];
  return a;
}

template <bool kM16>
__global__ void __launch_bounds__(kGvThreads, 1)
    nf4_gemv_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmX,
                    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    GemvArgs args) {
  extern __shared__ uint8_t gsm_raw[];
  uint32_t* table = reinterpret_cast<uint32_t*>(gsm_raw);
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(gsm_raw + kGvTable) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sB = ring + args.nstages * args.stage_bytes;      // B: rp rows x 256 columns bf16
  float* sc_ring = reinterpret_cast<float*>(sB + 512 * args.rp);   // [stage][4 blocks][128 rows]
  float* t8 = sc_ring + kGvMaxStages * kGvScaleWords;
  uint64_t* full = reinterpret_cast<uint64_t*>(t8 + 256);
  uint64_t* empty = full + kGvMaxStages;
  uint64_t* sfull = empty + kGvMaxStages;
  uint64_t* bfull = sfull + kGvMaxStages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  pdl_launch_dependents();
  if (threadIdx.x == kGvCompute * 32) {
    for (int s = 0; s < kGvMaxStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGvCompute);
      mbar_init(&sfull[s], 1);
    }
    mbar_init(bfull, 1);
    fence_mbar_init();
  }
  __syncthreads();   // the barriers are initialised
  if (warp != kGvCompute) {
    // Tables of constants (no global memory another launch writes), built by
    // every warp but the producer, which meanwhile starts the first copies:
    // entry e of the pair table is bf16(C[e >> 4]) | bf16(C[e & 15]) << 16,
    // one copy per bank; then T8.
    const int wi = warp < kGvCompute ? warp : warp - 1;
    const float cv = kCodeVals[16 * args.sv.codebook + (lane & 15)];
    for (int e = wi; e < 256; e += kGvWarps - 1)
      table[e * 64 + lane] =
          pack_bf16x2(__shfl_sync(0xFFFFFFFFu, cv, e >> 4), __shfl_sync(0xFFFFFFFFu, cv, e & 15));
    for (int u = wi * 32 + lane; u < 256; u += (kGvWarps - 1) * 32) t8[u] = kT8Table.v[u];
    asm volatile("bar.sync 2, %0;" ::"n"((kGvWarps - 1) * 32) : "memory");
  }

  const int M = args.M, N = args.N, K = args.K;
  const int cg = blockIdx.x;                            // 256-column group
  const int split = blockIdx.y, S = gridDim.y;          // the cluster spans all of y
  const int nk = (K + kGvRows - 1) / kGvRows;
  const int st0 = split * args.stages_per_split;
  const int nst = max(0, min(nk, st0 + args.stages_per_split) - st0);
  const bool zc_only = args.zc_only != 0;
  const uint32_t ring0 = smem_u32(ring);
  bool ok = true;

  if (warp == kGvCompute) {
    // --------------------------------- producer ---------------------------------
    pdl_wait();
    if (lane == 0) {
      if (!zc_only) tma_prefetch_desc(&tmP);
      tma_prefetch_desc(&tmX);
      tma_prefetch_desc(&tmA);
      if (!zc_only) {
        tma_prefetch_desc(&tmB);
        mbar_arrive_expect_tx(bfull, static_cast<uint32_t>(512 * args.rp));
        tma_load_2d(sB, &tmB, bfull, cg * kGvCols, 0);
      }
      const uint32_t tx = (zc_only ? 0u : static_cast<uint32_t>(kGvPk)) + kGvXb +
                          static_cast<uint32_t>(kGvRows * args.rp2 * 2);
      uint32_t last_parity[kGvMaxStages];
#pragma unroll
      for (int s = 0; s < kGvMaxStages; ++s) last_parity[s] = 2;
      auto issue = [&](int j, int s, uint32_t ph) {
        const int k0 = (st0 + j) * kGvRows;
        uint8_t* base = ring + s * args.stage_bytes;
        mbar_arrive_expect_tx(&full[s], tx);
        if (!zc_only) tma_load_2d(base, &tmP, &full[s], cg * 128, k0);
        tma_load_2d(base + kGvPk, &tmX, &full[s], k0, 0);
        tma_load_2d(base + kGvPk + 2048, &tmX, &full[s], k0 + 64, 0);
        tma_load_2d(base + kGvPk + kGvXb, &tmA, &full[s], 0, k0);
        last_parity[s] = ph;
      };
      const int ns = args.nstages;
      for (int j = 0; j < nst && j < ns; ++j) issue(j, j, 0);
      int s = 0;
      uint32_t ph = 0;
      for (int j = 0; j + ns < nst; ++j) {
        if (!mbar_wait(&empty[s], ph)) { ok = false; break; }
        issue(j + ns, s, ph ^ 1);
        if (++s == ns) { s = 0; ph ^= 1; }
      }
      // every copy issued has landed before the ring is reused or the CTA exits
      for (int q = 0; q < ns; ++q)
        if (last_parity[q] < 2 && !mbar_wait(&full[q], last_parity[q])) ok = false;
      if (!zc_only && !mbar_wait(bfull, 0)) ok = false;
    }
  } else if (warp > kGvCompute) {
    // ------------------------------- scale warps ------------------------------
    // a'[row][block] of every stage into sc_ring[stage][block][row].  Scale
    // warp q takes the stages q, q + kGvScaleWarps, ...; lane l decodes block
    // l & 3 for rows (l >> 2) + 8i, i < 16, and keeps its next stage's raw
    // loads in flight while it decodes this one, kGvScaleWarps stages ahead
    // of the compute warps.
    pdl_wait();
    const int sq = warp - kGvCompute - 1;
    if (!zc_only) {
      const int b = lane & 3, rl = lane >> 2;
      const int blk = cg * 4 + b;
      const bool colok = blk * 64 < N;
      const int bpr = N / 64;
      const bool dq = args.sv.code8 != nullptr;
      const float off = dq ? __ldg(args.sv.offset) : 0.0f;
      uint32_t qv[16];
      float fv[16];
      auto load = [&](int j) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int row = (st0 + j) * kGvRows + rl + 8 * i;
          qv[i] = 0u;
          fv[i] = 0.0f;
          if (colok && row < K) {
            const GvScale z = gemv_scale_load(args.sv, static_cast<int64_t>(row) * bpr + blk);
            qv[i] = z.q;
            fv[i] = z.v;
          }
        }
      };
      if (sq < nst) load(sq);
      for (int j = sq; j < nst; j += kGvScaleWarps) {
        const int s = j % args.nstages;
        const uint32_t ph = static_cast<uint32_t>((j / args.nstages) & 1);
        float a[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          a[i] = dq ? __fadd_rn(__fmul_rn(t8[qv[i]], fv[i]), off) : fv[i];
        if (j + kGvScaleWarps < nst) load(j + kGvScaleWarps);
        // the compute warps are done with this slot's previous stage
        if (j >= args.nstages && !mbar_wait(&empty[s], ph ^ 1)) { ok = false; break; }
        float* dst = sc_ring + s * kGvScaleWords + b * kGvRows + rl;
#pragma unroll
        for (int i = 0; i < 16; ++i) dst[8 * i] = a[i];
        __syncwarp();
        if (lane == 0) mbar_arrive(&sfull[s]);
      }
    }
  } else {
    // ------------------------------ compute warps ------------------------------
    pdl_wait();
    const int b = warp & 3, p = warp >> 2;             // column block, row slot
    const int blk = cg * 4 + b;                        // 64-column block
    const bool colok = !zc_only && blk * 64 < N;
    const int g = lane >> 2, t = lane & 3;
    const int kb = 16 * p;                             // rows kb.. and kb+64.. of a stage
    const uint32_t tbase = smem_u32(gsm_raw);
    const uint32_t laneword = lane * 4;
    // Packed stage (128-byte swizzle: row R at R*128, 16-byte chunk c at
    // (c ^ (R & 7))*16): this lane reads the 4 bytes of columns 8g..8g+7 of
    // block b in rows kb+2t, kb+2t+1 and the same rows +8 (+1024 bytes).
    const uint32_t cw = static_cast<uint32_t>(2 * b + (g >> 2));
    const uint32_t wo = static_cast<uint32_t>((g & 3) * 4);
    const uint32_t r0 = static_cast<uint32_t>(kb + 2 * t);
    const uint32_t poff0 = r0 * 128 + ((cw ^ (r0 & 7)) << 4) + wo;
    const uint32_t poff1 = (r0 + 1) * 128 + ((cw ^ ((r0 + 1) & 7)) << 4) + wo;
    // X stage (two halves of 16 tokens x 64 k, 128-byte swizzle): token g,
    // k = kb + 2t (+1) and kb + 8 + 2t (+1); tokens g + 8 one KB on
    const uint32_t c0 = static_cast<uint32_t>(kb >> 3);
    const uint32_t xoff0 = kGvPk + g * 128 + ((c0 ^ static_cast<uint32_t>(g)) << 4) + t * 4;
    const uint32_t xoff1 = kGvPk + g * 128 + (((c0 + 1) ^ static_cast<uint32_t>(g)) << 4) + t * 4;
    // Rows of A (rp2 bf16 each, swizzled by the span rp2*2 bytes): rank tiles
    // jt = b and b + 4 of X·A belong to this warp; ldmatrix rows kb + (lane & 15)
    const int rtiles = (args.r + 7) >> 3;
    const int nzt = (b < rtiles ? 1 : 0) + (b + 4 < rtiles ? 1 : 0);
    uint32_t zoff[2] = {0u, 0u};
    {
      const int cpr = args.rp2 >> 3;                   // 16-byte chunks per row of A
      const int zsh = cpr == 8 ? 0 : (cpr == 4 ? 1 : (cpr == 2 ? 2 : 3));
      const int arow = kb + (lane & 15);
      const int sw = (arow >> zsh) & (cpr - 1);
#pragma unroll
      for (int i = 0; i < 2; ++i)
        zoff[i] = static_cast<uint32_t>(kGvPk + kGvXb + arow * args.rp2 * 2 + (((b + 4 * i) ^ sw) << 4));
    }
    const uint32_t ahalf = static_cast<uint32_t>(64 * args.rp2 * 2);   // A rows of the second step
    // this lane's decode scales: a'[block b][rows kb + 2t, +1] and [kb + 2t + 8, +9]
    const uint32_t soff = static_cast<uint32_t>((b * kGvRows + kb + 2 * t) * 4);
    const uint32_t sc0 = smem_u32(sc_ring);

    // acc[f]: fragment rows = weight columns 8g+2f (g) and 8g+2f+1 (g+8),
    // columns = tokens 2t, 2t+1 (acc2: tokens 8+2t, 9+2t)
    float acc[4][4], acc2[4][4], zacc[2][4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[jj][i] = acc2[jj][i] = 0.0f;
#pragma unroll
    for (int jj = 0; jj < 2; ++jj)
#pragma unroll
      for (int i = 0; i < 4; ++i) zacc[jj][i] = 0.0f;

    // one 16-row step h (0: rows kb.., 1: rows kb+64..) of the stage at `sb`
    auto step = [&](uint32_t sb, uint32_t ss, int h) {
      const uint32_t xs = sb + static_cast<uint32_t>(2048 * h);
      const uint32_t x0 = lds32(xs + xoff0), x1 = lds32(xs + xoff1);
      uint32_t y0 = 0u, y1 = 0u;
      if (kM16) {
        y0 = lds32(xs + xoff0 + 1024);
        y1 = lds32(xs + xoff1 + 1024);
      }
      if (colok) {
        const uint32_t ps = sb + static_cast<uint32_t>(8192 * h);
        const uint32_t w0 = lds32(ps + poff0), w8 = lds32(ps + poff0 + 1024);
        const uint32_t w1 = lds32(ps + poff1), w9 = lds32(ps + poff1 + 1024);
        float2 sa, sbv;
        asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(sa.x), "=f"(sa.y) : "r"(ss + 256 * h));
        asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(sbv.x), "=f"(sbv.y) : "r"(ss + 256 * h + 32));
        // B fragments: scaled activations of token g (and g + 8)
        const uint32_t bx0 =
            pack_bf16x2(__uint_as_float(x0 << 16) * sa.x, __uint_as_float(x0 & 0xFFFF0000u) * sa.y);
        const uint32_t bx1 =
            pack_bf16x2(__uint_as_float(x1 << 16) * sbv.x, __uint_as_float(x1 & 0xFFFF0000u) * sbv.y);
        uint32_t by0 = 0u, by1 = 0u;
        if (kM16) {
          by0 = pack_bf16x2(__uint_as_float(y0 << 16) * sa.x, __uint_as_float(y0 & 0xFFFF0000u) * sa.y);
          by1 = pack_bf16x2(__uint_as_float(y1 << 16) * sbv.x, __uint_as_float(y1 & 0xFFFF0000u) * sbv.y);
        }
        // bytes (row k nibble, row k+1 nibble) per column: even and odd columns
        const uint32_t lo_e = (w0 & 0xF0F0F0F0u) | ((w1 >> 4) & 0x0F0F0F0Fu);
        const uint32_t lo_o = ((w0 << 4) & 0xF0F0F0F0u) | (w1 & 0x0F0F0F0Fu);
        const uint32_t hi_e = (w8 & 0xF0F0F0F0u) | ((w9 >> 4) & 0x0F0F0F0Fu);
        const uint32_t hi_o = ((w8 << 4) & 0xF0F0F0F0u) | (w9 & 0x0F0F0F0Fu);
#pragma unroll
        for (int f = 0; f < 4; ++f) {
          // address (byte f << 8) | lane*4: output byte 0 <- lane*4 (source
          // byte 4), byte 1 <- byte f of the word, bytes 2, 3 <- 0 (byte 5)
          const uint32_t sel = 0x5504u | (static_cast<uint32_t>(f) << 4);
          uint32_t wa[4];
          wa[0] = lds32(tbase + prmt(lo_e, laneword, sel));   // column 8g+2f, k 2t..
          wa[1] = lds32(tbase + prmt(lo_o, laneword, sel));   // column 8g+2f+1
          wa[2] = lds32(tbase + prmt(hi_e, laneword, sel));   // column 8g+2f, k 2t+8..
          wa[3] = lds32(tbase + prmt(hi_o, laneword, sel));
          mma_bf16_16816(acc[f], wa, bx0, bx1);
          if (kM16) mma_bf16_16816(acc2[f], wa, by0, by1);
        }
      }
      // X·A: raw activations (tokens as rows) against A[k][8 jt + g]
      const uint32_t araw[4] = {x0, y0, x1, y1};
      if (nzt > 0) {
        uint32_t zb0, zb1;
        ldsm_x2_trans(sb + zoff[0] + ahalf * h, zb0, zb1);
        mma_bf16_16816(zacc[0], araw, zb0, zb1);
        if (nzt > 1) {
          ldsm_x2_trans(sb + zoff[1] + ahalf * h, zb0, zb1);
          mma_bf16_16816(zacc[1], araw, zb0, zb1);
        }
      }
    };

    int s = 0;
    uint32_t ph = 0;
    for (int j = 0; j < nst; ++j) {
      if (!mbar_wait(&full[s], ph) || (colok && !mbar_wait(&sfull[s], ph))) { ok = false; break; }
      const uint32_t sb = ring0 + static_cast<uint32_t>(s * args.stage_bytes);
      const uint32_t ss = sc0 + static_cast<uint32_t>(s * kGvScaleWords * 4) + soff;
      step(sb, ss, 0);
      step(sb, ss, 1);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (++s == args.nstages) { s = 0; ph ^= 1; }
    }
    // every compute warp is past its last stage (and the producer has seen every
    // copy land) before the ring is reused for the sums
    asm volatile("bar.sync 1, %0;" ::"n"(kGvCompute * 32) : "memory");
    float* red = reinterpret_cast<float*>(ring + kGvRedOff);
    float* zred = reinterpret_cast<float*>(ring + kGvZredOff);
    float* Ps = reinterpret_cast<float*>(ring + kGvPsOff);
    float* Zs = reinterpret_cast<float*>(ring + kGvZsOff);
    if (p > 0) {
      float* myr = red + ((p - 1) * 4 + b) * 1024;
#pragma unroll
      for (int f = 0; f < 4; ++f)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          myr[(4 * f + q) * 32 + lane] = acc[f][q];
          if (kM16) myr[(16 + 4 * f + q) * 32 + lane] = acc2[f][q];
        }
      float* myz = zred + ((p - 1) * 4 + b) * 256;
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int q = 0; q < 4; ++q) myz[(4 * i + q) * 32 + lane] = zacc[i][q];
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kGvCompute * 32) : "memory");
    if (p == 0) {
      // the four row slots of block b, in slot order, into this CTA's sums
#pragma unroll
      for (int f = 0; f < 4; ++f)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col = b * 64 + 8 * g + 2 * f + (q >> 1);
          const int tok = 2 * t + (q & 1);
          const int i = 4 * f + q;
          float v = acc[f][q];
#pragma unroll
          for (int pp = 0; pp < 3; ++pp) v += red[(pp * 4 + b) * 1024 + i * 32 + lane];
          if (tok < M) Ps[tok * kGvPLd + col] = v;
          if (kM16) {
            float v2 = acc2[f][q];
#pragma unroll
            for (int pp = 0; pp < 3; ++pp) v2 += red[(pp * 4 + b) * 1024 + (16 + i) * 32 + lane];
            if (tok + 8 < M) Ps[(tok + 8) * kGvPLd + col] = v2;
          }
        }
#pragma unroll
      for (int i = 0; i < 2; ++i)
        if (i < nzt)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float v = zacc[i][q];
#pragma unroll
            for (int pp = 0; pp < 3; ++pp) v += zred[(pp * 4 + b) * 256 + (4 * i + q) * 32 + lane];
            const int tok = g + 8 * (q >> 1);
            const int jr = 8 * (b + 4 * i) + 2 * t + (q & 1);
            if (tok < M) Zs[tok * 64 + jr] = v;
          }
    }
  }

  // ---- the cluster's sums, in split order, through distributed shared memory
  cluster_sync_all();
  {
    const float* Zs = reinterpret_cast<const float*>(ring + kGvZsOff);
    const float* Ps = reinterpret_cast<const float*>(ring + kGvPsOff);
    float* Zcs = reinterpret_cast<float*>(ring + kGvZcOff);
    const int r = args.r;
    const bool writer = cg == 0 && split == 0;
    for (int e = threadIdx.x; e < M * 64; e += blockDim.x) {
      const int m = e >> 6, jr = e & 63;
      float zc = 0.0f;
      uint16_t bits = 0;
      if (jr < r) {
        const uint32_t off = smem_u32(Zs + m * 64 + jr);
        const float a = cluster_sum_in_order(off, S);
        bits = static_cast<uint16_t>(pack_bf16x2(args.c * a, 0.0f) & 0xFFFFu);
        zc = bf16_bits_to_f32(bits);
      }
      Zcs[e] = zc;
      if (writer && jr < args.ldz) args.Zc[static_cast<int64_t>(m) * args.ldz + jr] = bits;
    }
    __syncthreads();
    if (!zc_only) {
      // this CTA's share of the group's columns: Y = bf16(sums + Zc·B)
      const int share = (kGvCols + S - 1) / S;
      const int cl0 = split * share, ncl = max(0, min(kGvCols, cl0 + share) - cl0);
      const uint16_t* Bs = reinterpret_cast<const uint16_t*>(sB);
      for (int e = threadIdx.x; e < M * ncl; e += blockDim.x) {
        const int tok = e / ncl, cl = cl0 + (e - tok * ncl);
        const int n = cg * kGvCols + cl;
        if (n >= N) continue;
        const uint32_t off = smem_u32(Ps + tok * kGvPLd + cl);
        const float y = cluster_sum_in_order(off, S);
        float lora = 0.0f;
        for (int jr = 0; jr < r; ++jr)
          lora = fmaf(Zcs[tok * 64 + jr], bf16_bits_to_f32(Bs[jr * kGvCols + cl]), lora);
        args.Y[static_cast<int64_t>(tok) * N + n] =
            static_cast<uint16_t>(pack_bf16x2(y + lora, 0.0f) & 0xFFFFu);
      }
    }
  }
  cluster_sync_all();   // no CTA leaves while another still reads its sums
  if (!ok && lane == 0) raise_status(args.d_status, QLORA_ERR_TIMEOUT);
}

constexpr CUtensorMapSwizzle swizzle_for_bytes(int row_bytes) {
  return row_bytes >= 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : (row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                             : (row_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                                : CU_TENSOR_MAP_SWIZZLE_NONE));
}

int pow2_at_least8(int v) {
  int p = 8;
  while (p < v) p <<= 1;
  return p;
}



// Smem bytes besides the stage ring: the pair table (+ alignment slack), the
// B tile, the decode-scale ring, T8 and the barriers.
int gemv_fixed_smem(int rp) {
  return kGvTable + 1024 + 512 * rp + kGvMaxStages * kGvScaleWords * 4 + 256 * 4 + 256;
}

// Clusters of 1 x S x 1 CTAs (one per SM at this kernel's shared memory)
// that can be resident at once on this device, S = 1 .. 8; 0 if none.
struct ClusterFit {
  int n[9];
};

ClusterFit cluster_fit(int dev) {
  static ClusterFit fit[kMaxDevices];
  static DeviceOnce once;
  const cudaError_t e = once.run([](int d) {
    ClusterFit f{};
    for (int S = 1; S <= 8; ++S) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(1, static_cast<unsigned>(S), 1);
      cfg.blockDim = dim3(kGvThreads);
      cfg.dynamicSmemBytes = static_cast<size_t>(kGvSmemMax);
      cudaLaunchAttribute a[1];
      a[0].id = cudaLaunchAttributeClusterDimension;
      a[0].val.clusterDim.x = 1;
      a[0].val.clusterDim.y = static_cast<unsigned>(S);
      a[0].val.clusterDim.z = 1;
      cfg.attrs = a;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, nf4_gemv_kernel<false>, &cfg) != cudaSuccess) n = 0;
      f.n[S] = n;
    }
    (void)cudaGetLastError();
    fit[d] = f;
    return cudaSuccess;
  });
  ClusterFit none{};
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) return none;
  return fit[dev];
}

}  // namespace

// K splits: stage-granular ranges.  Among the cluster sizes S whose G
// clusters (one per 256-column group) are all resident at once (one wave),
// take the one with the fewest stages per CTA (the fewest S on a tie).  The
// plan depends only on K, N and the device, so the forward and the backward's
// recompute of Zc use the same splits.
GemvPlan gemv_plan(int64_t K, int64_t N, int num_sms) {
  GemvPlan pl;
  pl.G = static_cast<int>((N + kGvCols - 1) / kGvCols);
  const int nk = static_cast<int>((K + kGvRows - 1) / kGvRows);
  int dev = 0;
  const ClusterFit fit = cudaGetDevice(&dev) == cudaSuccess ? cluster_fit(dev) : ClusterFit{};
  int bestS = 1, best = nk;
  for (int S = 2; S <= 8 && S <= nk; ++S) {
    const int resident = fit.n[S] > 0 ? fit.n[S] : num_sms / S;
    if (pl.G > resident) continue;
    const int per = (nk + S - 1) / S;
    if (per < best) {
      best = per;
      bestS = S;
    }
  }
  pl.per = (nk + bestS - 1) / bestS;
  pl.S = (nk + pl.per - 1) / pl.per;
  return pl;
}

cudaError_t launch_gemv(int64_t M, int64_t K, int64_t N, int r, const uint16_t* X,
                        const uint8_t* packed, ScaleView sv, const uint16_t* A_pad, int rp,
                        const uint16_t* B, float c, uint16_t* Y, uint16_t* Zc, int ldz,
                        bool zc_only, int32_t* d_status, cudaStream_t st, int num_sms) {
  static DeviceOnce once;
  cudaError_t e = once.run([](int) {
    cudaError_t a = cudaFuncSetAttribute(nf4_gemv_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kGvSmemMax);
    if (a == cudaSuccess)
      a = cudaFuncSetAttribute(nf4_gemv_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kGvSmemMax);
    return a;
  });
  if (e != cudaSuccess) return e;
  const GemvPlan pl = gemv_plan(K, N, num_sms);
  GemvArgs ga;
  ga.M = static_cast<int>(M);
  ga.K = static_cast<int>(K);
  ga.N = static_cast<int>(N);
  ga.r = r;
  ga.rp = rp;
  ga.rp2 = pow2_at_least8(rp);
  ga.stage_bytes = kGvPk + kGvXb + kGvRows * ga.rp2 * 2;
  const int fixed = gemv_fixed_smem(rp);
  ga.nstages = (kGvSmemMax - fixed) / ga.stage_bytes;
  if (ga.nstages > kGvMaxStages) ga.nstages = kGvMaxStages;
  if (ga.nstages < 2 || ga.nstages * ga.stage_bytes < kGvEpilogueBytes) return cudaErrorInvalidValue;
  ga.stages_per_split = pl.per;
  ga.zc_only = zc_only ? 1 : 0;
  ga.c = c;
  ga.sv = sv;
  ga.Y = Y;
  ga.Zc = Zc;
  ga.ldz = ldz;
  ga.d_status = d_status;
  const size_t smem = static_cast<size_t>(fixed) + static_cast<size_t>(ga.nstages) * ga.stage_bytes;

  constexpr CUtensorMapDataType kBF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap tP, tX, tA, tB;
  if (!make_tmap_2d(&tP, packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, N / 2, N / 2, 128, kGvRows,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tX, X, kBF16, 2, M, K, K, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tA, A_pad, kBF16, 2, K, rp, rp, ga.rp2, kGvRows, swizzle_for_bytes(ga.rp2 * 2)))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tB, B, kBF16, 2, r, N, N, kGvCols, rp, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(zc_only ? 1 : pl.G), static_cast<unsigned>(pl.S));
  {
    ProfScope prof(zc_only ? kProfSkinny : kProfGemv, st);
    if (M <= 8)
      e = launch_pdl(nf4_gemv_kernel<false>, grid, dim3(kGvThreads), smem, st, pl.S, tP, tX, tA, tB, ga);
    else
      e = launch_pdl(nf4_gemv_kernel<true>, grid, dim3(kGvThreads), smem, st, pl.S, tP, tX, tA, tB, ga);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace qnf4
