/*
 * qlora_nf4.h — C ABI of the NF4 frozen-base LoRA linear layer for NVIDIA
 * B200 (sm_100a).
 *
 * The layer (page "QLoRA：冻结的 4-bit 权重怎样参与一次微调", §量化基座与可训练支路
 * 怎样相加 and §冻结权重为什么仍然需要输入梯度):
 *
 *     Z = X·A,   Y = X·Ŵ + c·Z·B               X: M×K, Ŵ: K×N, A: K×r, B: r×N
 *     dZ = c·G·Bᵀ,  dX = G·Ŵᵀ + dZ·Aᵀ,  dA = Xᵀ·dZ,  dB = c·Zᵀ·G
 *
 * where Ŵ is decoded on the fly from blockwise NF4 codes and G = ∂L/∂Y.
 * No gradient is produced for Ŵ or its packed codes and scales.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers named d_* or documented as "device" are CUDA device pointers;
 *   everything else (the state struct itself, scalars, the status output of
 *   qlora_status_sync) is host memory.
 * - All matrices are dense, row-major and contiguous.  bf16 tensors are passed
 *   as uint16_t bit patterns.  Device pointers must be 16-byte aligned.
 * - Ownership: the caller allocates and frees every buffer, including the
 *   workspace whose size the *_workspace_size functions report.  The library
 *   never allocates device memory and never synchronizes the stream, except
 *   in qlora_status_sync.
 * - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default).
 *   qlora_linear_bwd forks part of its work onto a library stream and joins
 *   it back before returning (see there).
 * - Errors: a host-side validation failure returns its qlora_status at once and
 *   enqueues nothing.  Errors that only the device can see (non-finite input,
 *   bad padding, an internal wait that ran out) are OR-ed as bit (1 << code)
 *   into the caller's device word `d_status` (may be NULL to ignore them) and
 *   the kernel finishes normally; outputs are then unspecified.  Read the word
 *   with qlora_status_sync and clear it with qlora_status_clear.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* qlora_stream_t;   /* same type as cudaStream_t */

typedef int32_t qlora_status;
#define QLORA_OK               0
#define QLORA_ERR_INVALID_ARG  1   /* null pointer, bad size, misaligned buffer, small workspace */
#define QLORA_ERR_UNSUPPORTED  2   /* shape outside the supported set (see each call) */
#define QLORA_ERR_NONFINITE    3   /* NaN/Inf weight or non-finite reconstruction */
#define QLORA_ERR_BAD_PADDING  4   /* odd-length payload whose last low nibble is not code 7 */
#define QLORA_ERR_CUDA         5   /* a CUDA runtime call failed (no device, launch error) */
#define QLORA_ERR_TIMEOUT      6   /* a bounded device-side wait ran out */

typedef int32_t qlora_dtype;
#define QLORA_DTYPE_BF16 0
#define QLORA_DTYPE_F32  1

/*
 * Quantized state of one K×N weight (page "QLoRA：冻结的 4-bit 权重怎样参与一次
 * 微调", §从 NF4 索引打包成字节 and §Double Quantization 压缩的是 Scale).
 *
 * The weight is flattened row-major (index i = k·N + n) and cut into blocks
 * of 64 consecutive elements; block b holds elements [64b, 64b+64), the last
 * one possibly shorter.  n1 = ceil(numel/64), n2 = ceil(n1/256).
 *   packed : ceil(numel/2) bytes; byte i = (code[2i] << 4) | code[2i+1]; an odd
 *            tail is padded with code 7 in the low nibble.           (device)
 *   absmax : n1 fp32 first-level scales, used when double_quant == 0. (device)
 *   code8  : n1 8-bit codes of the centred scales (double_quant == 1). (device)
 *   s2     : n2 fp32 second-level scales (double_quant == 1).          (device)
 *   offset : 1 fp32, the mean of the first-level scales (double_quant == 1).
 *            Decode scale a' = (T8[code8[b]] · s2[b/256]) + offset, each
 *            operation rounded to fp32.                                (device)
 * Unused pointers may be NULL.  The struct itself lives in host memory.
 *
 * codebook selects the 16 code values:
 *   QLORA_CODEBOOK_NF4  : the NF4 table; odd-tail padding code 7.
 *   QLORA_CODEBOOK_INT4 : uniform signed INT4, the comparator type of page
 *     "SFT（四）：QLoRA的4-bit量化与LoRA微调原理", §6 先理解最普通的分块量化:
 *     code j holds q = j - 8 (the quantizer emits 1 .. 15: q = clip(round(w/s),
 *     -7, 7), w/s in fp64, ties away from zero); `absmax` then holds the stored
 *     scale s = RN_fp32(amax/7) (1 for an all-zero block); padding code 8;
 *     double_quant must be 0 (else QLORA_ERR_UNSUPPORTED).
 * Every kernel of the library decodes both: w_hat = RN_bf16(value(code) · scale).
 */
#define QLORA_CODEBOOK_NF4  0
#define QLORA_CODEBOOK_INT4 1
typedef struct qlora_nf4_state {
  int64_t  numel;         /* logical element count (K·N for a weight), >= 1 */
  int32_t  blocksize;     /* must be 64 */
  int32_t  double_quant;  /* 0 or 1 */
  int32_t  dq_blocksize;  /* must be 256 */
  int32_t  codebook;      /* QLORA_CODEBOOK_NF4 (0) or QLORA_CODEBOOK_INT4 (1) */
  uint8_t* packed;
  float*   absmax;
  uint8_t* code8;
  float*   s2;
  float*   offset;
} qlora_nf4_state;

/* ABI version of this header (bumped on any incompatible change). */
#define QLORA_NF4_ABI_VERSION 2
int32_t qlora_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* qlora_status_str(qlora_status s);

/* For diagnostics: the description of the CUDA runtime error behind the
 * calling thread's most recent QLORA_ERR_CUDA (a static string from the CUDA
 * runtime, never NULL), or "no error" if this thread has had none. */
const char* qlora_last_cuda_error(void);

/* Element counts: n1 = ceil(numel/64), n2 = ceil(n1/256); 0 for numel < 1. */
int64_t qlora_nf4_n1(int64_t numel);
int64_t qlora_nf4_n2(int64_t numel);

/*
 * Read the device status word on `stream` (this call synchronizes the stream)
 * into *h_mask (host) and return the lowest-numbered error whose bit is set,
 * or QLORA_OK.  Returns QLORA_ERR_CUDA if the copy fails.
 */
qlora_status qlora_status_sync(const int32_t* d_status, qlora_stream_t stream, int32_t* h_mask);

/* Enqueue a reset of the device status word to 0. */
qlora_status qlora_status_clear(int32_t* d_status, qlora_stream_t stream);

/*
 * NF4 quantization — page "QLoRA：冻结的 4-bit 权重怎样参与一次微调",
 * §NF4 保存的是索引而不是均匀整数值, §从 NF4 索引打包成字节 and
 * §Double Quantization 压缩的是 Scale.
 *
 * Per 64-block: a = max|w| (exact), scale s = a, or 1 for an all-zero block;
 * code = the index of the nearest of the 16 NF4 values to w/s, ties to the
 * smaller index (decided exactly, as real numbers); codes packed high nibble
 * first.  Without double quantization s goes to st->absmax.  With it, the
 * n1 scales are centred on their exactly computed, once-rounded fp32 mean
 * (st->offset), cut into groups of 256 with an fp32 absmax each (st->s2; 1
 * for an all-zero group), and each centred scale gets the 8-bit code of the
 * nearest value of the signed dynamic codebook T8 (ties to the smaller value)
 * in st->code8.  The codes always come from the exact first-level scale.
 *
 *   W        : device, numel elements of `dtype` (QLORA_DTYPE_BF16 or _F32).
 *   st       : host struct; numel >= 1; its device buffers receive the result.
 *   ws       : device workspace of at least
 *              qlora_nf4_quantize_workspace_size(numel, double_quant) bytes
 *              (may be NULL when that size is 0); any contents on entry (the
 *              call clears what it uses itself, on the device).
 * Device errors: QLORA_ERR_NONFINITE if any weight is NaN or ±Inf.
 * Host errors: INVALID_ARG (null/misaligned pointers, numel < 1, bad
 * blocksize, small workspace), UNSUPPORTED (numel > 2^40), CUDA.
 */
size_t qlora_nf4_quantize_workspace_size(int64_t numel, int32_t double_quant);
qlora_status qlora_nf4_quantize(const void* W, qlora_dtype dtype, const qlora_nf4_state* st,
                                void* ws, size_t ws_bytes, int32_t* d_status,
                                qlora_stream_t stream);

/*
 * Sharded quantization for data-parallel replicas (page "SFT（四）：QLoRA的
 * 4-bit量化与LoRA微调原理", §26.1 为什么微批次设为 1: the effective batch spans
 * devices, each holding the same frozen base).  Each of several processes
 * encodes a contiguous range [block_begin, block_end) of the 64-blocks; the
 * ranges together must cover 0 .. n1 exactly once.  The result, once the
 * pieces are exchanged, is bit-identical to qlora_nf4_quantize of the whole
 * tensor.
 *
 *   1. qlora_nf4_quantize_shard_begin: W_shard points at element
 *      block_begin * 64 of the weight (the elements up to block_end * 64, or
 *      to numel for the last block).  Writes the packed bytes of the range
 *      into st->packed (at byte block_begin * 32) and, without double
 *      quantization, the scales into st->absmax[block_begin ..].  With
 *      double quantization the range's scales go to ws, and the first 2048
 *      bytes of ws receive 256 unsigned 64-bit sums (exponent bins of the
 *      range's scales).
 *   2. The caller adds those 256 sums element-wise over every shard (an
 *      integer all-reduce: exact, in any order) and writes the totals back
 *      into the first 2048 bytes of each shard's ws.
 *   3. qlora_nf4_quantize_shard_end (double quantization only; otherwise a
 *      no-op): from the total bins, st->offset (the exact mean of all n1
 *      scales, the same on every shard), and the scale codes and s2 of the
 *      range's groups (st->code8[block_begin ..], st->s2[block_begin/256 ..]).
 *   4. The caller gathers each shard's packed bytes, code8 and s2 (or
 *      absmax) ranges into every replica.
 * With double quantization block_begin must be a multiple of 256 and
 * block_end a multiple of 256 or n1 (whole groups per shard), else
 * INVALID_ARG.  An empty range (block_begin == block_end) is allowed anywhere
 * (begin clears the bins; end forms only the offset).  st describes the whole tensor (numel = K·N); its
 * buffers are full-size.  ws: at least qlora_nf4_quantize_shard_workspace_size
 * bytes, the same buffer for begin and end (0 bytes without DQ).
 */
size_t qlora_nf4_quantize_shard_workspace_size(int64_t numel_total, int64_t block_begin,
                                               int64_t block_end, int32_t double_quant);
qlora_status qlora_nf4_quantize_shard_begin(const void* W_shard, qlora_dtype dtype,
                                            const qlora_nf4_state* st, int64_t block_begin,
                                            int64_t block_end, void* ws, size_t ws_bytes,
                                            int32_t* d_status, qlora_stream_t stream);
qlora_status qlora_nf4_quantize_shard_end(const qlora_nf4_state* st, int64_t block_begin,
                                          int64_t block_end, const void* ws, size_t ws_bytes,
                                          int32_t* d_status, qlora_stream_t stream);

/*
 * Allocation-free NF4 quantization (no counterpart on the pages: it is a
 * property of this library, not of the method).  Same computation, arguments
 * and errors as qlora_nf4_quantize, without the workspace: some callers cannot
 * allocate device memory when they quantize (runtimes that plan every device
 * buffer at start-up and forbid allocation in their steady state; plugins that
 * only receive tensor pointers from a host framework).  The scratch it needs
 * (2304 bytes of exponent bins, a counter and a call token, plus one fp32 per
 * 64-block;
 * about 4 MB at the limit) is a
 * fixed array inside the library, allocated on each GPU that loads this part
 * of the library and held until the process exits.
 *   - numel must not exceed QLORA_NOALLOC_MAX_NUMEL, else QLORA_ERR_UNSUPPORTED.
 *   - The first call on a device, made with that device current, looks up the
 *     scratch's device address; make that first call before any stream
 *     capture.
 *   - All calls share the one scratch array (cleared where it must start at
 *     zero by each call): calls that overlap on the GPU, from any stream or
 *     thread, race with each other.  Serialize them.
 */
#define QLORA_NOALLOC_MAX_NUMEL (1ll << 26)
qlora_status qlora_nf4_quantize_noalloc(const void* W, qlora_dtype dtype,
                                        const qlora_nf4_state* st, int32_t* d_status,
                                        qlora_stream_t stream);

/*
 * NF4 dequantization — page "QLoRA：冻结的 4-bit 权重怎样参与一次微调",
 * §NF4 保存的是索引而不是均匀整数值 (reconstruction a·C_j) and §量化基座与可训练
 * 支路怎样相加 (BF16 compute type).
 *
 * W_hat[i] = bf16(C[code_i] · a'_b), the exact product rounded once to bf16
 * (nearest, ties to even), a'_b the decode scale of block b = i/64.
 *   W_hat : device, numel bf16 outputs.
 * Device errors: BAD_PADDING (odd numel whose last low nibble is not 7),
 * NONFINITE (a decode scale that is not finite).
 */
qlora_status qlora_nf4_dequantize(const qlora_nf4_state* st, uint16_t* W_hat,
                                  int32_t* d_status, qlora_stream_t stream);

/*
 * Forward — Z = X·A, Y = X·Ŵ + c·Z·B (page "QLoRA：冻结的 4-bit 权重怎样参与一次
 * 微调", §量化基座与可训练支路怎样相加; c = α/r).
 *
 *   X  : device bf16 M×K      A : device bf16 K×r      B : device bf16 r×N
 *   W  : NF4 state of the K×N weight (numel must equal K·N)
 *   Y  : device bf16 M×N output
 *   Zc : device bf16 M×r output, bf16(c·X·A); pass it to qlora_linear_bwd.
 * The product is computed in fp32 on bf16 operands and Ŵ is never written to
 * memory.  M > 16 runs the fused tensor-core path: Ŵ is decoded in tiles to
 * bf16, each weight within one bf16 ulp of qlora_nf4_dequantize's output.
 * M <= 16 runs the HBM-bound GEMV path, which folds each block's decode scale
 * into the activation instead: every product is bf16(x·a')·bf16(C_j), one
 * more bf16 rounding (relative <= 2^-9) than x·Ŵ carries; measured on the
 * 4096 x 11008 and 11008 x 4096 decode shapes, Y is within 3.7e-3 relative
 * Frobenius error of the fp64 result (the bf16 output rounding included).
 * Shapes: M >= 1, K % 64 == 0, N % 64 == 0, 1 <= r <= 64, else UNSUPPORTED.
 * A rank that is not a multiple of 8 is zero-padded to the next multiple of 8
 * inside the workspace (A, and the copy of Zc the tensor-core path reads), so
 * that every row the tensor maps read starts on a 16-byte boundary; the padded
 * rank columns are zero and change no result.
 * ws: at least qlora_linear_fwd_workspace_size(M, K, N, r) bytes; that size is
 * 0 when r % 8 == 0 (the kernels of the forward keep their partial sums on
 * chip: K splits added inside a thread-block cluster, or a whole contraction
 * in one CTA), and ws may then be null.
 * Work placement (no effect on the results): for M > 16 the fused GEMM runs
 * on the fewest CTA pairs that keep its number of waves of tiles; when that
 * leaves at least 8 SMs and Zc is small enough for them, Zc is formed there
 * while the fused GEMM runs, else before it.
 */
size_t qlora_linear_fwd_workspace_size(int64_t M, int64_t K, int64_t N, int32_t r);
qlora_status qlora_linear_fwd(int64_t M, int64_t K, int64_t N, int32_t r,
                              const uint16_t* X, const qlora_nf4_state* W,
                              const uint16_t* A, const uint16_t* B, float c,
                              uint16_t* Y, uint16_t* Zc,
                              void* ws, size_t ws_bytes, int32_t* d_status,
                              qlora_stream_t stream);

/*
 * Backward — page "QLoRA：冻结的 4-bit 权重怎样参与一次微调",
 * §冻结权重为什么仍然需要输入梯度:
 *   dZ = c·dY·Bᵀ,   dX = dY·Ŵᵀ + dZ·Aᵀ,   dA = Xᵀ·dZ,   dB = Zcᵀ·dY  (= c·Zᵀ·dY)
 *
 *   dY : device bf16 M×N       X : device bf16 M×K
 *   Zc : the forward's Zc, or NULL: the call then recomputes bf16(c·X·A) with
 *        the forward's own kernel and split (bit-identical), so a chain of
 *        layers need not keep M×r per layer between its forward and backward
 *        (recompute instead of save, as gradient checkpointing trades
 *        recomputation for stored activations: page "SFT（四）：QLoRA的4-bit
 *        量化与LoRA微调原理", §26.2 为什么开启 Gradient Checkpointing; page
 *        "QLoRA：冻结的 4-bit 权重怎样参与一次微调", §Paged Optimizer 管理哪一部分内存)
 *   dX : device bf16 M×K output
 *   dA : device fp32 K×r output     dB : device fp32 r×N output
 * No gradient is produced for W (the frozen base).  Same shape rules and
 * workspace convention as the forward.
 * Streams: dA and dB run on a stream the library owns (one per device,
 * created on first use), forked from `stream` after dZ and joined back into
 * it before the call returns, so that they use the SMs that dX leaves free
 * (as in the forward, dZ too runs there when it is small enough).  To the caller the call is still one
 * operation ordered on `stream` (later work on `stream` sees dX, dA and dB;
 * it can be captured in a CUDA graph), and the results are the same bits as
 * a run in order.  If the library stream cannot be created, or while
 * rank-r launches are being timed (qlora_profile_*), everything runs in
 * order on `stream`.
 */
size_t qlora_linear_bwd_workspace_size(int64_t M, int64_t K, int64_t N, int32_t r);
qlora_status qlora_linear_bwd(int64_t M, int64_t K, int64_t N, int32_t r,
                              const uint16_t* dY, const uint16_t* X, const uint16_t* Zc,
                              const qlora_nf4_state* W, const uint16_t* A, const uint16_t* B,
                              float c, uint16_t* dX, float* dA, float* dB,
                              void* ws, size_t ws_bytes, int32_t* d_status,
                              qlora_stream_t stream);

/*
 * Merge / export — page "QLoRA：冻结的 4-bit 权重怎样参与一次微调",
 * §Merge 后还是不是训练时的函数: after training, the layer's function is Ŵ
 * together with the adapter; one delivery is the dense merged weight
 *   out = RN_bf16( Ŵ + c·A·B ),   Ŵ = RN_bf16(C_j·a') as qlora_nf4_dequantize.
 * The rank-r product is formed in fp32 (bf16 operands, fp32 accumulation) and
 * added to Ŵ in one fp32 fma before the single rounding to bf16, so each
 * output is within one bf16 ulp of the correctly rounded exact merge.  For
 * the re-quantized delivery, pass `out` to qlora_nf4_quantize (a new
 * quantization step: not the trained function in general).
 *   W   : NF4 state of the K×N weight (numel must equal K·N)
 *   A   : device bf16 K×r      B : device bf16 r×N     (row-major)
 *   out : device bf16 K×N output (may not alias A, B or the state)
 * Shapes as qlora_linear_fwd (K % 64 == 0, N % 64 == 0, 1 <= r <= 64).  A
 * non-finite decode scale raises QLORA_ERR_NONFINITE in d_status.
 * No workspace; asynchronous on `stream`.
 */
qlora_status qlora_nf4_merge(int64_t K, int64_t N, int32_t r, const qlora_nf4_state* W,
                             const uint16_t* A, const uint16_t* B, float c, uint16_t* out,
                             int32_t* d_status, qlora_stream_t stream);

/*
 * Self-test of failure detection (no counterpart on the pages).  Launches one
 * kernel that waits, with the library's bounded wait, on an mbarrier that
 * nothing completes; after `limit_ns` (1 ns .. 10 s) of wall time the wait
 * gives up, QLORA_ERR_TIMEOUT is OR-ed into *d_status and the kernel returns.
 * Every wait inside the library's kernels is bounded the same way (2 s), so a
 * lost arrival surfaces as this status instead of a hang, and the context
 * stays usable.  Errors: INVALID_ARG (limit out of range, null status), CUDA.
 */
qlora_status qlora_selftest_bounded_wait(int64_t limit_ns, int32_t* d_status, qlora_stream_t stream);

/*
 * Launch timing, for measurement tools (no counterpart on the pages).  While
 * enabled, each kernel launch of the library is bracketed by two CUDA events
 * recorded on the stream the kernel runs on.  qlora_profile_read waits for
 * the recorded events, adds their elapsed times to per-class totals and
 * returns the total milliseconds and the launch count of class `kind`
 * (QLORA_PROF_*), or of all classes for kind = -1.  Launch counts are kept
 * whether or not timing is enabled.  qlora_profile_reset zeroes the totals.
 * qlora_profile_select restricts timing to the classes whose bit is set in
 * `kinds_mask` (bit k = class k; all classes by default).  The events sit
 * between launches and so keep a timed launch from overlapping its
 * predecessor's tail (programmatic dependent launch): a measuring tool that
 * wants the untouched launch chain times only the classes it needs.  While
 * QLORA_PROF_SKINNY is timed, the backward runs dA and dB in order on the
 * caller's stream (not beside dX), so that the class times do not overlap.
 * Not thread-safe across devices; meant for one measuring process.
 */
#define QLORA_PROF_FUSED_FWD  0   /* fused NF4 GEMM, forward (Y)        */
#define QLORA_PROF_FUSED_BWD  1   /* fused NF4 GEMM, input gradient (dX) */
#define QLORA_PROF_SKINNY     2   /* rank-r contractions (Zc, dZ, dA, dB) */
#define QLORA_PROF_QUANTIZE   3   /* NF4 encoder and double quantization */
#define QLORA_PROF_DEQUANTIZE 4   /* standalone dequantization           */
#define QLORA_PROF_GEMV       5   /* M <= 16 GEMV                        */
#define QLORA_PROF_OTHER      6   /* GEMV split sums                     */
qlora_status qlora_profile_enable(int32_t on);
qlora_status qlora_profile_read(int32_t kind, double* total_ms, int64_t* launches);
qlora_status qlora_profile_reset(void);
qlora_status qlora_profile_select(uint32_t kinds_mask);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* QLORA_NF4_H */
