// Launchers of the library's kernels and device helpers shared between
// translation units.  Internal to the library (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <utility>

#include "common.cuh"

namespace qnf4 {

// One-time set-up per device (kernel attributes, occupancy queries).
// cudaFuncSetAttribute acts on the current device only, so every device that
// runs a kernel gets its own run of `f(dev)`; a failed run is retried on the
// next call.  Safe when several host threads make their first calls at once.
constexpr int kMaxDevices = 64;
class DeviceOnce {
 public:
  template <typename F>
  cudaError_t run(F&& f) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (done_[dev].load(std::memory_order_acquire)) return cudaSuccess;
    std::lock_guard<std::mutex> lock(mu_);
    if (done_[dev].load(std::memory_order_relaxed)) return cudaSuccess;
    e = f(dev);
    if (e == cudaSuccess) done_[dev].store(true, std::memory_order_release);
    return e;
  }

 private:
  std::mutex mu_;
  std::atomic<bool> done_[kMaxDevices] = {};
};

// The scale codebook T8 (see make_t8_table in common.cuh), one copy per
// translation unit in constant memory; build_t8 stages it in shared memory,
// where a warp's lookups of different codes do not serialize.
static __constant__ T8Table kT8Table = make_t8_table();

__device__ __forceinline__ void build_t8(float* t8 /*256*/) {
  for (int u = threadIdx.x; u < 256; u += blockDim.x) t8[u] = kT8Table.v[u];
}

// Launch with programmatic stream serialization (and, when cluster_y > 1, a
// thread-block cluster of 1 x cluster_y x 1).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, int cluster_y, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_y > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = 1;
    attr[n].val.clusterDim.y = static_cast<unsigned>(cluster_y);
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The same for a kernel whose CTA pairs share tensor-core products
// (cta_group::2): clusters of 2 x 1 x 1, the pair's CTAs adjacent in x.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_pair(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// selftest.cu — a wait that nothing completes, bounded by limit_ns
cudaError_t launch_bounded_wait_selftest(int32_t* d_status, uint64_t limit_ns, cudaStream_t st);

// quantize.cu.  With double quantization the workspace holds, from its
// start: 256 exponent bins of the scales (2 KB), the counter of finished
// encoder CTAs, the call's token, the flag of its mean and the counter of
// claimed chunks, then (at kQuantizeWsHead) one fp32 scale per 64-block; CTA
// 0 of every call resets the head (any contents on entry).
constexpr size_t kQuantizeWsHead = 2304;
cudaError_t launch_quantize(const void* W, int dtype, int64_t numel, uint8_t* packed,
                            float* absmax_out, bool dq, uint8_t* code8, float* s2, float* offset,
                            void* ws, int32_t* d_status, cudaStream_t st, int num_sms,
                            int codebook = 0);
size_t quantize_workspace_bytes(int64_t numel, bool dq);
// Sharded quantization (blocks [b0, b1) of a tensor of numel_total elements;
// W_shard points at element b0 * 64).  begin: packed bytes and, without DQ,
// the scales go straight into the full-size state; with DQ the shard's
// scales and the exponent bins of their sums go to `ws` (same layout as the
// quantize workspace).  end: with the bins holding the sum over every shard,
// the offset and the scale codes and s2 of the shard's groups.
cudaError_t launch_quantize_shard_begin(const void* W_shard, int dtype, int64_t numel_total,
                                        int64_t b0, int64_t b1, uint8_t* packed, float* absmax_out,
                                        bool dq, void* ws, int32_t* d_status, cudaStream_t st,
                                        int num_sms, int codebook);
cudaError_t launch_quantize_shard_end(int64_t numel_total, int64_t b0, int64_t b1, const void* ws,
                                      uint8_t* code8, float* s2, float* offset, cudaStream_t st,
                                      int num_sms);

// dequantize.cu
cudaError_t launch_dequantize(const uint8_t* packed, int64_t numel, const float* absmax,
                              const uint8_t* code8, const float* s2, const float* offset,
                              uint16_t* out, int32_t* d_status, cudaStream_t st, int num_sms,
                              int codebook = 0);

// Decode-scale view of a quantized weight, shared by the GEMM and GEMV paths.
struct ScaleView {
  int codebook;          // 0: NF4, 1: uniform INT4 (its stored scale is amax / 7)
  const float* absmax;   // non-null when not double-quantized
  const uint8_t* code8;  // non-null when double-quantized
  const float* s2;
  const float* offset;
};

// merge.cu — the merged dense weight RN_bf16(ŵ + c·A·B)
cudaError_t launch_merge(int64_t K, int64_t N, int r, float c, ScaleView sv, const uint8_t* packed,
                         const uint16_t* A, const uint16_t* B, uint16_t* out, int32_t* d_status,
                         cudaStream_t st);

// gemv.cu — the M <= 16 forward (and, with zc_only, the recompute of its Zc):
// A_pad is A with its rows padded to rp (a multiple of 8) columns; Zc is
// written with row pitch ldz (columns r .. ldz-1 as 0) by one CTA.
struct GemvPlan {
  int G;     // 256-column groups
  int S;     // K splits = cluster size
  int per;   // 128-row stages per split
};
GemvPlan gemv_plan(int64_t K, int64_t N, int num_sms);
cudaError_t launch_gemv(int64_t M, int64_t K, int64_t N, int r, const uint16_t* X,
                        const uint8_t* packed, ScaleView sv, const uint16_t* A_pad, int rp,
                        const uint16_t* B, float c, uint16_t* Y, uint16_t* Zc, int ldz,
                        bool zc_only, int32_t* d_status, cudaStream_t st, int num_sms);

// linear.cu — forward and backward of the layer
size_t linear_fwd_workspace_bytes(int64_t M, int64_t K, int64_t N, int r);
size_t linear_bwd_workspace_bytes(int64_t M, int64_t K, int64_t N, int r);
cudaError_t launch_linear_fwd(int64_t M, int64_t K, int64_t N, int r, const uint16_t* X,
                              const uint8_t* packed, ScaleView sv, const uint16_t* A,
                              const uint16_t* B, float c, uint16_t* Y, uint16_t* Zc, void* ws,
                              size_t ws_bytes, int32_t* d_status, cudaStream_t st, int num_sms);
cudaError_t launch_linear_bwd(int64_t M, int64_t K, int64_t N, int r, const uint16_t* dY,
                              const uint16_t* X, const uint16_t* Zc, const uint8_t* packed,
                              ScaleView sv, const uint16_t* A, const uint16_t* B, float c,
                              uint16_t* dX, float* dA, float* dB, void* ws, size_t ws_bytes,
                              int32_t* d_status, cudaStream_t st, int num_sms);

}  // namespace qnf4
