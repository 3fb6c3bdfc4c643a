// Standalone NF4 dequantization to bf16.  Page "QLoRA：冻结的 4-bit 权重怎样参与
// 一次微调", §NF4 保存的是索引而不是均匀整数值 (w = a·C_j) and §量化基座与可训练
// 支路怎样相加 (the decoded weight is consumed in BF16).
#include <cfloat>

#include "common.cuh"
#include "kernels.cuh"
#include "profile.cuh"

namespace qnf4 {

__constant__ float kNF4d[32] = {QNF4_TABLE_VALUES, QNF4_INT4_VALUES};   // NF4, INT4

// Per 64-block decode scale: absmax, or T8[q]*s2 + offset with each operation
// rounded to fp32 (no fusion).
__device__ __forceinline__ float decode_scale(int64_t blk, const float* __restrict__ absmax,
                                              const uint8_t* __restrict__ code8,
                                              const float* __restrict__ s2, float off,
                                              const float* t8) {
  if (code8 == nullptr) return __ldg(absmax + blk);
  const float v = t8[__ldg(code8 + blk)];
  return __fadd_rn(__fmul_rn(v, __ldg(s2 + (blk >> 8))), off);
}

// One thread per 8 consecutive weights (4 packed bytes -> one 16-byte store).
__global__ void __launch_bounds__(256) nf4_dequant_kernel(
    const uint8_t* __restrict__ packed, int64_t numel, const float* __restrict__ absmax,
    const uint8_t* __restrict__ code8, const float* __restrict__ s2,
    const float* __restrict__ offset, uint16_t* __restrict__ out, int32_t* d_status, int codebook) {
  __shared__ float C[16];
  __shared__ float t8[256];
  pdl_launch_dependents();
  if (threadIdx.x < 16) C[threadIdx.x] = kNF4d[16 * codebook + threadIdx.x];
  if (code8 != nullptr) build_t8(t8);
  __syncthreads();
  pdl_wait();   // the tables above read no global memory
  const float off = code8 != nullptr ? __ldg(offset) : 0.0f;
  const int64_t nbytes = (numel + 1) >> 1;
  const int64_t ngroups = (numel + 7) >> 3;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  bool nonfinite = false, badpad = false;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < ngroups;
       g += stride) {
    const int64_t e0 = g * 8;
    const float a = decode_scale(e0 >> 6, absmax, code8, s2, off, t8);
    nonfinite |= !(fabsf(a) <= FLT_MAX);
    const int64_t b0 = e0 >> 1;
    uint32_t word;
    const bool full = e0 + 8 <= numel;
    if (full) {
      word = __ldg(reinterpret_cast<const uint32_t*>(packed + b0));
    } else {
      word = 0x77777777u;
      for (int k = 0; k < 4; ++k)
        if (b0 + k < nbytes) {
          word &= ~(0xFFu << (8 * k));
          word |= static_cast<uint32_t>(__ldg(packed + b0 + k)) << (8 * k);
        }
      if ((numel & 1) && ((nbytes - 1) - b0) < 4) {
        const int k = static_cast<int>((nbytes - 1) - b0);
        badpad |= ((word >> (8 * k)) & 0xFu) != static_cast<uint32_t>(codebook ? kPadCodeInt4 : kPadCode);
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t byte = (word >> (8 * k)) & 0xFFu;
      const uint32_t lo = bf16_of_exact_product(C[byte >> 4], a);   // element 2k
      const uint32_t hi = bf16_of_exact_product(C[byte & 15u], a);  // element 2k+1
      o[k] = lo | (hi << 16);
    }
    if (full) {
      *reinterpret_cast<uint4*>(out + e0) = make_uint4(o[0], o[1], o[2], o[3]);
    } else {
      for (int i = 0; i < 8; ++i)
        if (e0 + i < numel) out[e0 + i] = static_cast<uint16_t>(o[i >> 1] >> ((i & 1) * 16));
    }
  }
  if (nonfinite) raise_status(d_status, QLORA_ERR_NONFINITE);
  if (badpad) raise_status(d_status, QLORA_ERR_BAD_PADDING);
}

cudaError_t launch_dequantize(const uint8_t* packed, int64_t numel, const float* absmax,
                              const uint8_t* code8, const float* s2, const float* offset,
                              uint16_t* out, int32_t* d_status, cudaStream_t st, int num_sms,
                              int codebook) {
  const int threads = 256;
  const int64_t ngroups = (numel + 7) >> 3;
  const int64_t want = (ngroups + threads - 1) / threads;
  const int blocks = static_cast<int>(want < num_sms * 8LL ? want : num_sms * 8LL);
  {
    ProfScope prof(kProfDequantize, st);
    const cudaError_t e = launch_pdl(nf4_dequant_kernel, dim3(blocks), dim3(threads), 0, st, 1, packed,
                                     numel, absmax, code8, s2, offset, out, d_status, codebook);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace qnf4
