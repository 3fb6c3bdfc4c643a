// Shared device helpers for the sm_100a kernels: status word, NF4 table,
// bf16 helpers, and thin inline-PTX wrappers for mbarrier, TMA and tcgen05.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "qlora_nf4.h"

namespace qnf4 {

constexpr int kBlock = 64;     // first-level NF4 block
constexpr int kDQBlock = 256;  // second-level block of the scale codes
constexpr int kPadCode = 7;    // odd-tail padding code (exact zero)
constexpr int kPadCodeInt4 = 8;   // the same for the uniform INT4 codebook (q = 0)

// The 16 NF4 reconstruction values as printed on the page "QLoRA：冻结的
// 4-bit 权重怎样参与一次微调" (§从 NF4 索引打包成字节).  Every value is an exact
// fp32 number.
#define QNF4_TABLE_VALUES                                                        \
  -1.0f, -0.6961928009986877f, -0.5250730514526367f, -0.39491748809814453f,     \
      -0.28444138169288635f, -0.18477343022823334f, -0.09105003625154495f, 0.0f, \
      0.07958029955625534f, 0.16093020141124725f, 0.24611230194568634f,         \
      0.33791524171829224f, 0.44070982933044434f, 0.5626170039176941f,          \
      0.7229568362236023f, 1.0f

// The uniform signed INT4 codebook (page "SFT（四）：QLoRA的4-bit量化与LoRA微调原理",
// §6 先理解最普通的分块量化: w_hat = s·q, q in [-7, 7]): code j holds q = j - 8;
// the quantizer emits codes 1 .. 15 and pads an odd tail with code 8 (q = 0).
#define QNF4_INT4_VALUES                                                         \
  -8.0f, -7.0f, -6.0f, -5.0f, -4.0f, -3.0f, -2.0f, -1.0f, 0.0f, 1.0f, 2.0f, 3.0f, \
      4.0f, 5.0f, 6.0f, 7.0f

// The signed dynamic 8-bit codebook T8 of the scale codes (this library's own
// definition; the page only requires "a signed dynamic 8-bit codebook, not
// FP8 E4M3"): byte u, sign u >> 7, t = u & 127; t = 0 is 0; otherwise
// f = floor(log2 t), e = 6 - f, m = t - 2^f and |v| = (2^f + 9(m+1)) /
// (10^(e+1) 2^f), a correctly rounded double division rounded to fp32.
// Evaluated by the compiler (IEEE double division, then round to nearest
// float) into a table that decoding kernels copy from constant memory.
struct T8Table {
  float v[256];
};

constexpr double t8_pow10(int e) {
  double p = 10.0;
  for (int i = 0; i < e; ++i) p *= 10.0;
  return p;
}

constexpr float t8_value(int u) {
  const int t = u & 127;
  if (t == 0) return 0.0f;
  int f = 0;
  while ((2 << f) <= t) ++f;
  const int e = 6 - f, m = t - (1 << f);
  const float mag = static_cast<float>(static_cast<double>((1 << f) + 9 * (m + 1)) /
                                       (t8_pow10(e) * static_cast<double>(1 << f)));
  return (u >> 7) ? -mag : mag;
}

constexpr T8Table make_t8_table() {
  T8Table t{};
  for (int u = 0; u < 256; ++u) t.v[u] = t8_value(u);
  return t;
}
static_assert(make_t8_table().v[0x43] == 0.15625f && make_t8_table().v[0x7F] == 1.0f &&
                  make_t8_table().v[0xFF] == -1.0f && make_t8_table().v[0x80] == 0.0f,
              "T8 spot values");

// Raise an error bit in the caller's device status word.
__device__ __forceinline__ void raise_status(int32_t* d_status, int code) {
  if (d_status) atomicOr(d_status, 1 << code);
}

// max that propagates NaN (PTX max.NaN), used so that a NaN anywhere in a block
// reaches the block's absmax and is detected there.
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) {
  return __uint_as_float(b16 << 16);
}

// Two fp32 -> packed bf16x2 (lo in bits 0..15), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// bf16 rounding (nearest, ties to even) of the EXACT product c*a of two fp32
// numbers.  p = fl32(c*a) is one rounding away; the fma residual r = c*a - p
// is exact.  Rounding p again to bf16 can only go wrong when p sits exactly on
// a bf16 halfway point (low 16 bits 0x8000) while r != 0; moving p one fp32
// step towards the exact value then gives the single-rounding result.
__device__ __forceinline__ uint32_t bf16_of_exact_product(float c, float a) {
  float p = c * a;
  float r = fmaf(c, a, -p);
  uint32_t b = __float_as_uint(p);
  if ((b & 0xFFFFu) == 0x8000u && r != 0.0f) {
    b += ((__float_as_uint(r) ^ b) & 0x80000000u) ? 0xFFFFFFFFu : 1u;
  }
  float q = __uint_as_float(b);
  uint32_t out;
  asm("{ .reg .b16 h; cvt.rn.bf16.f32 h, %1; mov.b32 %0, {h, h}; }" : "=r"(out) : "f"(q));
  return out & 0xFFFFu;
}

// ---------------------------------------------------------------------------
// Shared-memory address, fences, mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// generic-proxy shared-memory writes -> visible to the async proxy (TMA, tcgen05)
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// try_wait suspends the calling thread until the phase completes or about
// `kSuspendNs` pass, so waiting warps do not spin on issue slots.
constexpr uint32_t kSuspendNs = 200000;

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Every wait on another agent is bounded: after `limit_ns` of wall time the
// wait gives up and returns false, and the caller unwinds and reports
// QLORA_ERR_TIMEOUT.  Correct code never comes close to the limit.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ bool mbar_wait_for(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < 4; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  return mbar_wait_for(bar, parity, kWaitLimitNs);
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  Every kernel of the library is launched
// with programmatic stream serialization: it lets its successor launch at once
// (pdl_launch_dependents at its start) and, before its first access to global
// memory that an earlier launch may write or read, waits for its predecessor
// to complete and flush (pdl_wait).  Only set-up that touches no such memory
// (shared memory, barriers, TMEM, tables of constants) runs before the wait.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// TMA (no multicast anywhere in this library)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// 1-D bulk copy global -> shared (no tensor map): both addresses 16-byte
// aligned, size a multiple of 16 bytes; completes `bytes` on `bar`.
__device__ __forceinline__ void bulk_load_1d(void* smem_dst, const void* gsrc, uint32_t bytes,
                                             uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// shared -> global tiled store (bulk-group completion); the tile's generic
// writes must be made visible to the async proxy first (fence_proxy_async_smem)
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int32_t x,
                                             int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(smem_src)), "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// wait until at most N committed bulk groups still READ their shared source
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// wait until at most N committed bulk groups are still in flight at all
template <int N>
__device__ __forceinline__ void bulk_wait_group() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------------------
// Thread-block clusters: a barrier over every thread of every CTA (lanes may
// arrive diverged), and a load from a peer CTA's shared memory at the same
// offset as `local_saddr` in this CTA.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

__device__ __forceinline__ float ld_dsmem_f32(uint32_t local_saddr, uint32_t cta_rank) {
  uint32_t remote;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_saddr), "r"(cta_rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

// ---------------------------------------------------------------------------
// tcgen05 (5th-generation tensor cores, accumulators in TMEM)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] x B[smem desc], kind::f16 (bf16 in, fp32 accumulate)
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when all tcgen05 operations issued so far by this
// thread have completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// The same as umma_commit, arriving on the barrier at the same shared-memory
// offset in every CTA of the cluster named in cta_mask (bit i = rank i).
__device__ __forceinline__ void umma_commit_mc(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

// Shared-memory address of the same offset in CTA `cta_rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t local_saddr, uint32_t cta_rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_saddr), "r"(cta_rank));
  return remote;
}

// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) from
// this CTA's shared memory to a peer CTA's (dst, a shared::cluster address),
// completing `bytes` on the peer's mbarrier (also a shared::cluster address).
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst, const void* src, uint32_t bytes,
                                                  uint32_t peer_bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "r"(smem_u32(src)), "r"(bytes), "r"(peer_bar)
      : "memory");
}

// ---------------------------------------------------------------------------
// CTA-pair (cta_group::2) forms: the two CTAs of a 2-CTA cluster share one
// TMEM allocation address and one MMA, issued by CTA rank 0, whose A operand
// is split by rows (M/2 per CTA) and B operand by columns (N/2 per CTA), both
// at the same shared-memory offset in each CTA; each CTA's TMEM receives its
// M/2 rows of D over all N columns.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the barrier at `bar`'s offset in every CTA named in cta_mask
// when all pair MMAs issued so far have completed.
__device__ __forceinline__ void umma_commit_pair_mc(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}
// Tiled TMA load into this CTA's shared memory whose completion is counted on
// an mbarrier that may live in the peer CTA of the pair (`bar_cluster`, a
// shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster, int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}
// Arrive on an mbarrier given by its shared::cluster address (this CTA's or
// the peer's).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}

// 32 lanes x 32 consecutive fp32 columns: thread t of the warp gets row
// (lane base + t), columns [col, col+32).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
        "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
        "=r"(v[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor (sm_100 UMMA): start address, leading and
// stride byte offsets (all >> 4), version 1, swizzle mode in bits 61..63.
constexpr uint64_t kSwizzle128B = 2;
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes,
                                              uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;                  // descriptor version for sm_100
  d |= kSwizzle128B << 61;          // 128-byte swizzle
  return d;
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 D, shape M x N.
// a_mn / b_mn select MN-major (1) or K-major (0) operand layouts.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                         // D format: F32
         | (1u << 7)                       // A format: BF16
         | (1u << 10)                      // B format: BF16
         | (static_cast<uint32_t>(a_mn) << 15) | (static_cast<uint32_t>(b_mn) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

}  // namespace qnf4
