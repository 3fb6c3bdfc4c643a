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
  const dim3 grid(static_cast<unsigned>(N / 64), static_cast<unsigned>((K + kMgRows - 1) / kMgRows));
  cudaError_t e;
  {
    ProfScope prof(kProfDequantize, st);
    e = launch_pdl(nf4_merge_kernel, grid, dim3(256), 0, st, 1, a);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace qnf4
