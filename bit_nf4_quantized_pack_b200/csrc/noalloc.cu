// qlora_nf4_quantize_noalloc: NF4 quantization (with or without double
// quantization) whose scratch memory is a fixed array compiled into the
// library instead of a caller-allocated workspace.
//
// Some callers cannot allocate device memory at the point where they quantize:
// runtimes that plan every device buffer at start-up and forbid allocation in
// their steady state (cudaMalloc may synchronize the device and fragments a
// fixed memory budget), and plugins that only receive tensor pointers from a
// host framework and have no allocator of their own.  This entry point needs
// nothing from them but the inputs and outputs.
//
// The scratch (2 KB of exponent bins for the exact mean and a counter, 2304
// bytes in all, plus one fp32 scale per 64-block) lives in this file's module, so it is allocated only once that
// module is loaded, and every GPU that loads it keeps it until the process
// exits.  Its device address is looked up once per device, on the first call
// made with that device current.
#include <cuda_runtime.h>

#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "kernels.cuh"
#include "qlora_nf4.h"

namespace {

constexpr int64_t kNoAllocMaxBlocks = QLORA_NOALLOC_MAX_NUMEL / 64;
constexpr size_t kNoAllocScratchBytes = qnf4::kQuantizeWsHead + static_cast<size_t>(kNoAllocMaxBlocks) * 4;

__device__ __align__(256) unsigned char g_quantize_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[64] = {};

// Device address of g_quantize_scratch on the current device (the host-side
// symbol is only a stand-in and must never be passed to a kernel).
cudaError_t scratch_on_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_quantize_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The same NVTX range as the library's other compute entry points.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

}  // namespace

extern "C" qlora_status qlora_nf4_quantize_noalloc(const void* W, qlora_dtype dtype,
                                                   const qlora_nf4_state* st, int32_t* d_status,
                                                   qlora_stream_t stream) {
  NvtxRange nvtx_range("qlora_nf4_quantize_noalloc");
  if (!st || !W || !aligned(W, 16)) return QLORA_ERR_INVALID_ARG;
  if (st->numel < 1 || st->blocksize != qnf4::kBlock) return QLORA_ERR_INVALID_ARG;
  if (st->codebook != QLORA_CODEBOOK_NF4 && st->codebook != QLORA_CODEBOOK_INT4) return QLORA_ERR_INVALID_ARG;
  if (st->double_quant != 0 && st->double_quant != 1) return QLORA_ERR_INVALID_ARG;
  if (st->codebook == QLORA_CODEBOOK_INT4 && st->double_quant) return QLORA_ERR_UNSUPPORTED;
  if (dtype != QLORA_DTYPE_BF16 && dtype != QLORA_DTYPE_F32) return QLORA_ERR_INVALID_ARG;
  if (!st->packed || !aligned(st->packed, 16)) return QLORA_ERR_INVALID_ARG;
  if (st->double_quant) {
    if (st->dq_blocksize != qnf4::kDQBlock || !st->code8 || !st->s2 || !st->offset)
      return QLORA_ERR_INVALID_ARG;
    if (!aligned(st->s2, 4) || !aligned(st->offset, 4)) return QLORA_ERR_INVALID_ARG;
  } else if (!st->absmax || !aligned(st->absmax, 4)) {
    return QLORA_ERR_INVALID_ARG;
  }
  if (st->numel > QLORA_NOALLOC_MAX_NUMEL) return QLORA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (scratch_on_current_device(&scratch) != cudaSuccess) return QLORA_ERR_CUDA;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return QLORA_ERR_CUDA;
  // the bins and the counter at the start of the scratch are cleared by the launcher
  cudaError_t e = qnf4::launch_quantize(W, dtype, st->numel, st->packed, st->absmax,
                                        st->double_quant != 0, st->code8, st->s2, st->offset,
                                        scratch, d_status,
                                        reinterpret_cast<cudaStream_t>(stream), sms, st->codebook);
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}
