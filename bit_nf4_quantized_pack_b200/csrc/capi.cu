// extern "C" boundary of the library: argument validation, workspace sizing,
// and dispatch to the kernels.  See include/qlora_nf4.h for the contract.
#include <cuda_runtime.h>
#include <stdint.h>

#include <cmath>

#include <nvtx3/nvToolsExt.h>

#include "kernels.cuh"
#include "qlora_nf4.h"

namespace {

constexpr int64_t kMaxNumel = (1ll << 38);

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev] = n;
  }
  return cached[dev];
}

// The CUDA error behind this thread's latest QLORA_ERR_CUDA (qlora_last_cuda_error).
thread_local cudaError_t t_last_cuda_error = cudaSuccess;

qlora_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return QLORA_OK;
  t_last_cuda_error = e;
  return QLORA_ERR_CUDA;
}

// An NVTX range around each compute entry point, so that a timeline tool
// shows the library's calls (header-only NVTX: no cost without a tool).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

// Common checks of a quantized-state struct.
qlora_status check_state(const qlora_nf4_state* st, bool need_scales) {
  if (!st) return QLORA_ERR_INVALID_ARG;
  if (st->numel < 1 || st->blocksize != qnf4::kBlock) return QLORA_ERR_INVALID_ARG;
  if (st->codebook != QLORA_CODEBOOK_NF4 && st->codebook != QLORA_CODEBOOK_INT4) return QLORA_ERR_INVALID_ARG;
  if (st->double_quant != 0 && st->double_quant != 1) return QLORA_ERR_INVALID_ARG;
  if (st->codebook == QLORA_CODEBOOK_INT4 && st->double_quant) return QLORA_ERR_UNSUPPORTED;
  if (st->numel > kMaxNumel) return QLORA_ERR_UNSUPPORTED;
  if (!st->packed || !aligned(st->packed, 16)) return QLORA_ERR_INVALID_ARG;
  if (!need_scales) return QLORA_OK;
  if (st->double_quant) {
    if (st->dq_blocksize != qnf4::kDQBlock) return QLORA_ERR_INVALID_ARG;
    if (!st->code8 || !st->s2 || !st->offset) return QLORA_ERR_INVALID_ARG;
    if (!aligned(st->s2, 4) || !aligned(st->offset, 4)) return QLORA_ERR_INVALID_ARG;
  } else {
    if (!st->absmax || !aligned(st->absmax, 4)) return QLORA_ERR_INVALID_ARG;
  }
  return QLORA_OK;
}

qnf4::ScaleView view_of(const qlora_nf4_state* st) {
  qnf4::ScaleView v{};
  v.codebook = st->codebook;
  if (st->double_quant) {
    v.code8 = st->code8;
    v.s2 = st->s2;
    v.offset = st->offset;
  } else {
    v.absmax = st->absmax;
  }
  return v;
}

qlora_status check_linear_shape(int64_t M, int64_t K, int64_t N, int32_t r) {
  if (M < 1 || K < 1 || N < 1) return QLORA_ERR_INVALID_ARG;
  if (K % 64 != 0 || N % 64 != 0) return QLORA_ERR_UNSUPPORTED;
  if (r < 1 || r > 64) return QLORA_ERR_UNSUPPORTED;
  if (M > (1ll << 30) || K > (1ll << 30) || N > (1ll << 30)) return QLORA_ERR_UNSUPPORTED;
  if (K * N > kMaxNumel) return QLORA_ERR_UNSUPPORTED;
  return QLORA_OK;
}

}  // namespace

extern "C" {

int32_t qlora_abi_version(void) { return QLORA_NF4_ABI_VERSION; }

const char* qlora_last_cuda_error(void) {
  return t_last_cuda_error == cudaSuccess ? "no error" : cudaGetErrorString(t_last_cuda_error);
}

const char* qlora_status_str(qlora_status s) {
  switch (s) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_INVALID_ARG: return "invalid argument";
    case QLORA_ERR_UNSUPPORTED: return "unsupported shape or option";
    case QLORA_ERR_NONFINITE: return "non-finite weight or reconstruction";
    case QLORA_ERR_BAD_PADDING: return "payload padding code is not 7";
    case QLORA_ERR_CUDA: return "CUDA runtime error";
    case QLORA_ERR_TIMEOUT: return "bounded device wait ran out";
    default: return "unknown status";
  }
}

int64_t qlora_nf4_n1(int64_t numel) { return numel < 1 ? 0 : (numel + 63) / 64; }
int64_t qlora_nf4_n2(int64_t numel) { return numel < 1 ? 0 : (qlora_nf4_n1(numel) + 255) / 256; }

qlora_status qlora_status_sync(const int32_t* d_status, qlora_stream_t stream, int32_t* h_mask) {
  if (!d_status || !h_mask) return QLORA_ERR_INVALID_ARG;
  int32_t m = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  qlora_status r = cuda_status(cudaMemcpyAsync(&m, d_status, sizeof(m), cudaMemcpyDeviceToHost, s));
  if (r != QLORA_OK) return r;
  r = cuda_status(cudaStreamSynchronize(s));
  if (r != QLORA_OK) return r;
  *h_mask = m;
  for (int code = 1; code < 31; ++code)
    if (m & (1 << code)) return code;
  return QLORA_OK;
}

qlora_status qlora_status_clear(int32_t* d_status, qlora_stream_t stream) {
  if (!d_status) return QLORA_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(d_status, 0, sizeof(int32_t),
                                     reinterpret_cast<cudaStream_t>(stream)));
}

size_t qlora_nf4_quantize_workspace_size(int64_t numel, int32_t double_quant) {
  if (numel < 1) return 0;
  return qnf4::quantize_workspace_bytes(numel, double_quant != 0);
}

qlora_status qlora_nf4_quantize(const void* W, qlora_dtype dtype, const qlora_nf4_state* st,
                                void* ws, size_t ws_bytes, int32_t* d_status,
                                qlora_stream_t stream) {
  NvtxRange nvtx_range("qlora_nf4_quantize");
  qlora_status v = check_state(st, true);
  if (v != QLORA_OK) return v;
  if (!W || !aligned(W, 16)) return QLORA_ERR_INVALID_ARG;
  if (dtype != QLORA_DTYPE_BF16 && dtype != QLORA_DTYPE_F32) return QLORA_ERR_INVALID_ARG;
  const size_t need = qlora_nf4_quantize_workspace_size(st->numel, st->double_quant);
  if (need > 0 && (!ws || ws_bytes < need || !aligned(ws, 16))) return QLORA_ERR_INVALID_ARG;
  const int sms = sm_count();
  if (sms <= 0) return QLORA_ERR_CUDA;
  cudaError_t e = qnf4::launch_quantize(W, dtype, st->numel, st->packed, st->absmax,
                                        st->double_quant != 0, st->code8, st->s2, st->offset, ws,
                                        d_status, reinterpret_cast<cudaStream_t>(stream), sms,
                                        st->codebook);
  return cuda_status(e);
}

size_t qlora_nf4_quantize_shard_workspace_size(int64_t numel_total, int64_t block_begin,
                                               int64_t block_end, int32_t double_quant) {
  if (numel_total < 1 || block_begin < 0 || block_end < block_begin ||
      block_end > qlora_nf4_n1(numel_total) || !double_quant)
    return 0;
  return qnf4::kQuantizeWsHead + static_cast<size_t>(block_end - block_begin) * 4;
}

namespace {
qlora_status check_shard(const qlora_nf4_state* st, int64_t b0, int64_t b1) {
  qlora_status v = check_state(st, true);
  if (v != QLORA_OK) return v;
  const int64_t n1 = qlora_nf4_n1(st->numel);
  if (b0 < 0 || b1 < b0 || b1 > n1) return QLORA_ERR_INVALID_ARG;
  // with double quantization a shard holds whole groups of 256 blocks (the
  // last shard may end at n1)
  if (st->double_quant && b1 > b0 &&
      (b0 % qnf4::kDQBlock != 0 || (b1 != n1 && b1 % qnf4::kDQBlock != 0)))
    return QLORA_ERR_INVALID_ARG;
  return QLORA_OK;
}
}  // namespace

qlora_status qlora_nf4_quantize_shard_begin(const void* W_shard, qlora_dtype dtype,
                                            const qlora_nf4_state* st, int64_t block_begin,
                                            int64_t block_end, void* ws, size_t ws_bytes,
                                            int32_t* d_status, qlora_stream_t stream) {
  NvtxRange nvtx_range("qlora_nf4_quantize_shard_begin");
  qlora_status v = check_shard(st, block_begin, block_end);
  if (v != QLORA_OK) return v;
  if (dtype != QLORA_DTYPE_BF16 && dtype != QLORA_DTYPE_F32) return QLORA_ERR_INVALID_ARG;
  const size_t need = qlora_nf4_quantize_shard_workspace_size(st->numel, block_begin, block_end,
                                                              st->double_quant);
  if (need > 0 && (!ws || ws_bytes < need || !aligned(ws, 16))) return QLORA_ERR_INVALID_ARG;
  if (block_end == block_begin) {
    // an empty shard contributes zero bins
    if (st->double_quant)
      return cuda_status(cudaMemsetAsync(ws, 0, qnf4::kQuantizeWsHead,
                                         reinterpret_cast<cudaStream_t>(stream)));
    return QLORA_OK;
  }
  if (!W_shard || !aligned(W_shard, 16)) return QLORA_ERR_INVALID_ARG;
  const int sms = sm_count();
  if (sms <= 0) return QLORA_ERR_CUDA;
  return cuda_status(qnf4::launch_quantize_shard_begin(
      W_shard, dtype, st->numel, block_begin, block_end, st->packed, st->absmax,
      st->double_quant != 0, ws, d_status, reinterpret_cast<cudaStream_t>(stream), sms,
      st->codebook));
}

qlora_status qlora_nf4_quantize_shard_end(const qlora_nf4_state* st, int64_t block_begin,
                                          int64_t block_end, const void* ws, size_t ws_bytes,
                                          int32_t* d_status, qlora_stream_t stream) {
  NvtxRange nvtx_range("qlora_nf4_quantize_shard_end");
  (void)d_status;
  qlora_status v = check_shard(st, block_begin, block_end);
  if (v != QLORA_OK) return v;
  if (!st->double_quant) return QLORA_OK;   // nothing happens after the bins
  const size_t need = qlora_nf4_quantize_shard_workspace_size(st->numel, block_begin, block_end, 1);
  if (!ws || ws_bytes < need || !aligned(ws, 16)) return QLORA_ERR_INVALID_ARG;
  const int sms = sm_count();
  if (sms <= 0) return QLORA_ERR_CUDA;
  return cuda_status(qnf4::launch_quantize_shard_end(st->numel, block_begin, block_end, ws,
                                                     st->code8, st->s2, st->offset,
                                                     reinterpret_cast<cudaStream_t>(stream), sms));
}

qlora_status qlora_nf4_dequantize(const qlora_nf4_state* st, uint16_t* W_hat, int32_t* d_status,
                                  qlora_stream_t stream) {
  NvtxRange nvtx_range("qlora_nf4_dequantize");
  qlora_status v = check_state(st, true);
  if (v != QLORA_OK) return v;
  if (!W_hat || !aligned(W_hat, 16)) return QLORA_ERR_INVALID_ARG;
  const int sms = sm_count();
  if (sms <= 0) return QLORA_ERR_CUDA;
  const qnf4::ScaleView sv = view_of(st);
  cudaError_t e = qnf4::launch_dequantize(st->packed, st->numel, sv.absmax, sv.code8, sv.s2,
                                          sv.offset, W_hat, d_status,
                                          reinterpret_cast<cudaStream_t>(stream), sms, sv.codebook);
  return cuda_status(e);
}

size_t qlora_linear_fwd_workspace_size(int64_t M, int64_t K, int64_t N, int32_t r) {
  if (check_linear_shape(M, K, N, r) != QLORA_OK) return 0;
  return qnf4::linear_fwd_workspace_bytes(M, K, N, r);
}

size_t qlora_linear_bwd_workspace_size(int64_t M, int64_t K, int64_t N, int32_t r) {
  if (check_linear_shape(M, K, N, r) != QLORA_OK) return 0;
  return qnf4::linear_bwd_workspace_bytes(M, K, N, r);
}

qlora_status qlora_linear_fwd(int64_t M, int64_t K, int64_t N, int32_t r, const uint16_t* X,
                              const qlora_nf4_state* W, const uint16_t* A, const uint16_t* B,
                              float c, uint16_t* Y, uint16_t* Zc, void* ws, size_t ws_bytes,
                              int32_t* d_status, qlora_stream_t stream) {
  NvtxRange nvtx_range("qlora_linear_fwd");
  qlora_status v = check_linear_shape(M, K, N, r);
  if (v != QLORA_OK) return v;
  v = check_state(W, true);
  if (v != QLORA_OK) return v;
  if (W->numel != K * N) return QLORA_ERR_INVALID_ARG;
  if (!std::isfinite(c)) return QLORA_ERR_INVALID_ARG;
  const void* ptrs[] = {X, A, B, Y, Zc};
  for (const void* p : ptrs)
    if (!p || !aligned(p, 16)) return QLORA_ERR_INVALID_ARG;
  const size_t need = qlora_linear_fwd_workspace_size(M, K, N, r);
  if (need > 0 && (!ws || ws_bytes < need || !aligned(ws, 16))) return QLORA_ERR_INVALID_ARG;
  const int sms = sm_count();
  if (sms <= 0) return QLORA_ERR_CUDA;
  cudaError_t e = qnf4::launch_linear_fwd(M, K, N, r, X, W->packed, view_of(W), A, B, c, Y, Zc,
                                          ws, ws_bytes, d_status,
                                          reinterpret_cast<cudaStream_t>(stream), sms);
  return cuda_status(e);
}

qlora_status qlora_nf4_merge(int64_t K, int64_t N, int32_t r, const qlora_nf4_state* W,
                             const uint16_t* A, const uint16_t* B, float c, uint16_t* out,
                             int32_t* d_status, qlora_stream_t stream) {
  NvtxRange nvtx_range("qlora_nf4_merge");
  qlora_status v = check_linear_shape(1, K, N, r);
  if (v != QLORA_OK) return v;
  v = check_state(W, true);
  if (v != QLORA_OK) return v;
  if (W->numel != K * N) return QLORA_ERR_INVALID_ARG;
  if (!std::isfinite(c)) return QLORA_ERR_INVALID_ARG;
  const void* ptrs[] = {A, B, out};
  for (const void* p : ptrs)
    if (!p || !aligned(p, 16)) return QLORA_ERR_INVALID_ARG;
  return cuda_status(qnf4::launch_merge(K, N, r, c, view_of(W), W->packed, A, B, out, d_status,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

qlora_status qlora_selftest_bounded_wait(int64_t limit_ns, int32_t* d_status, qlora_stream_t stream) {
  NvtxRange nvtx_range("qlora_selftest_bounded_wait");
  if (limit_ns < 1 || limit_ns > 10000000000ll || !d_status) return QLORA_ERR_INVALID_ARG;
  return cuda_status(qnf4::launch_bounded_wait_selftest(d_status, static_cast<uint64_t>(limit_ns),
                                                        reinterpret_cast<cudaStream_t>(stream)));
}

qlora_status qlora_linear_bwd(int64_t M, int64_t K, int64_t N, int32_t r, const uint16_t* dY,
                              const uint16_t* X, const uint16_t* Zc, const qlora_nf4_state* W,
                              const uint16_t* A, const uint16_t* B, float c, uint16_t* dX,
                              float* dA, float* dB, void* ws, size_t ws_bytes, int32_t* d_status,
                              qlora_stream_t stream) {
  NvtxRange nvtx_range("qlora_linear_bwd");
  qlora_status v = check_linear_shape(M, K, N, r);
  if (v != QLORA_OK) return v;
  v = check_state(W, true);
  if (v != QLORA_OK) return v;
  if (W->numel != K * N) return QLORA_ERR_INVALID_ARG;
  if (!std::isfinite(c)) return QLORA_ERR_INVALID_ARG;
  const void* ptrs[] = {dY, X, A, B, dX, dA, dB};
  for (const void* p : ptrs)
    if (!p || !aligned(p, 16)) return QLORA_ERR_INVALID_ARG;
  if (Zc && !aligned(Zc, 16)) return QLORA_ERR_INVALID_ARG;   // null: recompute it
  const size_t need = qlora_linear_bwd_workspace_size(M, K, N, r);
  if (need > 0 && (!ws || ws_bytes < need || !aligned(ws, 16))) return QLORA_ERR_INVALID_ARG;
  const int sms = sm_count();
  if (sms <= 0) return QLORA_ERR_CUDA;
  cudaError_t e = qnf4::launch_linear_bwd(M, K, N, r, dY, X, Zc, W->packed, view_of(W), A, B, c,
                                          dX, dA, dB, ws, ws_bytes, d_status,
                                          reinterpret_cast<cudaStream_t>(stream), sms);
  return cuda_status(e);
}

}  // extern "C"
