// NF4 encoder (absmax, nearest code, nibble pack) and double quantization of
// the block scales.  Page "QLoRA：冻结的 4-bit 权重怎样参与一次微调",
// §NF4 保存的是索引而不是均匀整数值, §从 NF4 索引打包成字节,
// §Double Quantization 压缩的是 Scale.
#include <cfloat>

#include "common.cuh"
#include "kernels.cuh"
#include "profile.cuh"

namespace qnf4 {

__constant__ float kNF4c[16] = {QNF4_TABLE_VALUES};

// ---------------------------------------------------------------------------
// Nearest-code search.
//
// The rule is: code = argmin_j |w/s - C_j| with ties to the smaller index.
// Since the table is sorted, that equals the number of midpoints
// m_j = (C_j + C_{j+1})/2 strictly below w/s, i.e. #{j : w > s*m_j} (s > 0).
// The fast path computes t = w * (1/s) in fp32 (absolute error < 2^-22) and
// looks t up in 33 uniform buckets of width 1/16 that are offset by half a
// bucket; every bucket holds at most one midpoint and no midpoint lies within
// 0.004 of a bucket edge, so a bucket gives (number of midpoints below it,
// the midpoint inside it).  Only when t is within 2^-20 of that midpoint is
// the comparison redone exactly: w > s*m_j in fp64, where s*m_j is exact
// (24-bit times at most 26-bit significand).  An exact tie (w == s*m_j) is
// not "greater", so it keeps the smaller index.
// ---------------------------------------------------------------------------
struct Bucket {
  float mid;  // the midpoint inside this bucket, or 4.0 (none)
  int jlo;    // number of midpoints below the bucket = code left of `mid`
};

constexpr int kBuckets = 33;
constexpr float kNearEps = 9.5367431640625e-07f;  // 2^-20

__device__ __forceinline__ void build_buckets(Bucket* tab, double* mexact) {
  for (int b = threadIdx.x; b < kBuckets; b += blockDim.x) {
    const double lo = (b - 16.5) / 16.0, hi = (b - 15.5) / 16.0;
    int jlo = 0;
    float mid = 4.0f;
    for (int j = 0; j < 15; ++j) {
      const double mj = 0.5 * (static_cast<double>(kNF4c[j]) + static_cast<double>(kNF4c[j + 1]));
      if (mj < lo)
        ++jlo;
      else if (mj < hi)
        mid = static_cast<float>(mj);
    }
    tab[b].mid = mid;
    tab[b].jlo = jlo;
  }
  for (int j = threadIdx.x; j < 15; j += blockDim.x)
    mexact[j] = 0.5 * (static_cast<double>(kNF4c[j]) + static_cast<double>(kNF4c[j + 1]));
}

__device__ __forceinline__ uint32_t nearest_code(float x, float s, float inv_s, const Bucket* tab,
                                                 const double* mexact) {
  const float t = x * inv_s;
  int b = __float2int_rd(fmaf(t, 16.0f, 16.5f));
  b = min(max(b, 0), kBuckets - 1);
  const Bucket e = tab[b];
  const float d = t - e.mid;
  uint32_t code = static_cast<uint32_t>(e.jlo) + (d > 0.0f ? 1u : 0u);
  if (fabsf(d) < kNearEps) {
    const double thr = static_cast<double>(s) * mexact[e.jlo];
    code = static_cast<uint32_t>(e.jlo) + (static_cast<double>(x) > thr ? 1u : 0u);
  }
  return code;
}

template <typename T>
__device__ __forceinline__ void load8(const T* __restrict__ W, int64_t e0, int64_t numel, bool vec,
                                      float (&x)[8]);

template <>
__device__ __forceinline__ void load8<uint16_t>(const uint16_t* __restrict__ W, int64_t e0,
                                                int64_t numel, bool vec, float (&x)[8]) {
  if (vec && e0 + 8 <= numel) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(W + e0));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      x[i] = (e0 + i < numel) ? bf16_bits_to_f32(__ldg(W + e0 + i)) : 0.0f;
  }
}

template <>
__device__ __forceinline__ void load8<float>(const float* __restrict__ W, int64_t e0, int64_t numel,
                                             bool vec, float (&x)[8]) {
  if (vec && e0 + 8 <= numel) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(W + e0));
    const float4 b = __ldg(reinterpret_cast<const float4*>(W + e0 + 4));
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = (e0 + i < numel) ? __ldg(W + e0 + i) : 0.0f;
  }
}

// One group of 8 lanes per 64-block; each lane owns 8 consecutive elements.
template <typename T, bool kDQ>
__global__ void __launch_bounds__(256) nf4_encode_kernel(const T* __restrict__ W, int64_t numel,
                                                         int64_t n1, uint8_t* __restrict__ packed,
                                                         float* __restrict__ scales,
                                                         unsigned long long* __restrict__ bins,
                                                         int32_t* d_status) {
  __shared__ Bucket tab[kBuckets];
  __shared__ double mexact[15];
  __shared__ unsigned long long sbins[kDQ ? 256 : 1];
  build_buckets(tab, mexact);
  if (kDQ)
    for (int i = threadIdx.x; i < 256; i += blockDim.x) sbins[i] = 0ull;
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int sub = lane & 7;
  const unsigned gmask = 0xFFu << (lane & 24);
  const bool vec = (reinterpret_cast<uintptr_t>(W) & 15u) == 0;
  const int64_t nbytes = (numel + 1) >> 1;
  const int64_t ngroups = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 3;
  bool bad = false;

  for (int64_t blk = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 3; blk < n1;
       blk += ngroups) {
    const int64_t e0 = blk * kBlock + sub * 8;
    float x[8];
    load8<T>(W, e0, numel, vec, x);
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) am = fmax_nan(am, fabsf(x[i]));
    am = fmax_nan(am, __shfl_xor_sync(gmask, am, 1));
    am = fmax_nan(am, __shfl_xor_sync(gmask, am, 2));
    am = fmax_nan(am, __shfl_xor_sync(gmask, am, 4));
    const bool finite = am <= FLT_MAX;
    bad |= !finite;
    const float s = (finite && am > 0.0f) ? am : 1.0f;
    // For a block scale below 2^-126, 1/s would overflow: scale the block and
    // its scale by 2^64 (exact for these tiny values) so the fast path stays
    // finite; codes depend only on the ratio w/s.
    const bool tiny = s < 1.17549435e-38f;
    const float sc = tiny ? 18446744073709551616.0f : 1.0f;
    const float s_eff = s * sc;
    const float inv_s = __frcp_rn(s_eff);
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t code = (finite && e0 + i < numel)
                                ? nearest_code(x[i] * sc, s_eff, inv_s, tab, mexact)
                                : kPadCode;
      // element 2k -> high nibble of byte k, element 2k+1 -> low nibble
      word |= code << ((i >> 1) * 8 + ((i & 1) ? 0 : 4));
    }
    const int64_t b0 = e0 >> 1;
    if (e0 + 8 <= numel) {
      *reinterpret_cast<uint32_t*>(packed + b0) = word;
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (b0 + k < nbytes) packed[b0 + k] = static_cast<uint8_t>(word >> (8 * k));
    }
    if (sub == 0) {
      scales[blk] = s;
      if (kDQ) {
        const uint32_t u = __float_as_uint(s);
        const uint32_t E = (u >> 23) & 0xFFu;
        const uint32_t mant = (u & 0x7FFFFFu) | (E ? 0x800000u : 0u);
        atomicAdd(&sbins[E ? E : 1u], static_cast<unsigned long long>(mant));
      }
    }
  }
  if (bad) raise_status(d_status, QLORA_ERR_NONFINITE);
  if (kDQ) {
    __syncthreads();
    for (int i = threadIdx.x; i < 256; i += blockDim.x)
      if (sbins[i]) atomicAdd(&bins[i], sbins[i]);
  }
}

// ---------------------------------------------------------------------------
// Exact mean of the first-level scales.  Scale s with biased exponent E and
// 24-bit integer mantissa q equals q * 2^(max(E,1) - 150); the encoder sums q
// per exponent (bins[max(E,1)], exact in 64 bits).  Here the bins are added
// into a 384-bit integer S in units of 2^-149, S is divided by n1 exactly
// (long division, quotient Q and remainder R) and Q + R/n1 is rounded once to
// fp32, to nearest with ties to even.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void add_u32_at(uint32_t* L, int nl, int i, uint32_t v) {
  uint64_t carry = v;
  for (; i < nl && carry; ++i) {
    const uint64_t t = static_cast<uint64_t>(L[i]) + carry;
    L[i] = static_cast<uint32_t>(t);
    carry = t >> 32;
  }
}

__device__ __forceinline__ int bit_of(const uint32_t* Q, int b) { return (Q[b >> 5] >> (b & 31)) & 1; }

// Round q * 2^e (q > 0 a 128-bit integer, plus an extra fraction rem/d of
// one unit 2^e, 0 <= rem < d) to the nearest fp32, ties to even.
__device__ uint32_t round_q128_to_f32(unsigned __int128 q, uint64_t rem, uint64_t d, int e) {
  if (q == 0) {
    // below one unit: only possible when 2^e is below the subnormal quantum
    // or the mean is exactly 0; scale up until the quantum is reached
    while (e > -149 && q == 0) {
      const unsigned __int128 t = static_cast<unsigned __int128>(rem) << 1;
      q = static_cast<unsigned __int128>(t / d);
      rem = static_cast<uint64_t>(t % d);
      --e;
    }
    if (q == 0) return 0u;
  }
  const uint64_t hi = static_cast<uint64_t>(q >> 64), lo = static_cast<uint64_t>(q);
  const int h = hi ? 127 - __clzll(static_cast<long long>(hi)) : 63 - __clzll(static_cast<long long>(lo));
  int qe = h + e - 23;                 // exponent of the fp32 quantum
  if (qe < -149) qe = -149;
  int shift = qe - e;
  if (shift < 0) {                     // make room below: bring fraction bits in
    const int up = -shift;
    const unsigned __int128 t = static_cast<unsigned __int128>(rem) << up;
    q = (q << up) + static_cast<unsigned __int128>(t / d);
    rem = static_cast<uint64_t>(t % d);
    shift = 0;
  }
  uint64_t mant = static_cast<uint64_t>(q >> shift);
  bool up;
  if (shift == 0) {
    up = (2 * rem > d) || (2 * rem == d && (mant & 1u));
  } else {
    const unsigned __int128 below = q & ((static_cast<unsigned __int128>(1) << shift) - 1);
    const unsigned __int128 half = static_cast<unsigned __int128>(1) << (shift - 1);
    up = below > half || (below == half && (rem != 0 || (mant & 1u)));
  }
  mant += up ? 1u : 0u;
  // value = mant * 2^qe with mant <= 2^24
  if (qe == -149 && mant < (1u << 23)) return static_cast<uint32_t>(mant);   // subnormal
  return (static_cast<uint32_t>(qe + 150) << 23) + static_cast<uint32_t>(mant - (1u << 23));
}

// One CTA of 256 threads: the bins are read in parallel, a warp ballot finds
// the occupied exponent range, and one thread adds the occupied bins exactly:
// in 128 bits when they span at most 64 binades (always, for any realistic
// weight), else in a 384-bit integer.
__global__ void __launch_bounds__(256) dq_mean_kernel(const unsigned long long* __restrict__ bins,
                                                      int64_t n1, float* __restrict__ offset) {
  __shared__ unsigned long long sb[256];
  __shared__ int range[2];
  sb[threadIdx.x] = bins[threadIdx.x];
  __syncthreads();
  if (threadIdx.x < 32) {
    uint32_t m = 0;
    for (int i = 0; i < 8; ++i) m |= (sb[threadIdx.x * 8 + i] != 0ull ? 1u : 0u) << i;
    const unsigned any = __ballot_sync(0xFFFFFFFFu, m != 0);
    const int lmin = __ffs(any) - 1, lmax = 31 - __clz(any);
    if (threadIdx.x == lmin) range[0] = threadIdx.x * 8 + (__ffs(m) - 1);
    if (threadIdx.x == lmax) range[1] = threadIdx.x * 8 + (31 - __clz(m));
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  const int kmin = range[0], kmax = range[1];
  const uint64_t d = static_cast<uint64_t>(n1);
  uint32_t bits;
  if (kmax - kmin <= 64) {
    unsigned __int128 S = 0;
    for (int key = kmin; key <= kmax; ++key)
      S += static_cast<unsigned __int128>(sb[key]) << (key - kmin);
    const unsigned __int128 Q = S / d;
    const uint64_t rem = static_cast<uint64_t>(S % d);
    bits = round_q128_to_f32(Q, rem, d, kmin - 1 - 149);
  } else {
    constexpr int NL = 12;
    uint32_t L[NL];
    for (int i = 0; i < NL; ++i) L[i] = 0;
    for (int key = kmin; key <= kmax; ++key) {
      const unsigned long long v = sb[key];
      if (!v) continue;
      const int sh = key - 1, li = sh >> 5, bi = sh & 31;
      const uint64_t p0 = (v & 0xFFFFFFFFull) << bi;
      const uint64_t p1 = (v >> 32) << bi;
      add_u32_at(L, NL, li, static_cast<uint32_t>(p0));
      add_u32_at(L, NL, li + 1, static_cast<uint32_t>(p0 >> 32));
      add_u32_at(L, NL, li + 1, static_cast<uint32_t>(p1));
      add_u32_at(L, NL, li + 2, static_cast<uint32_t>(p1 >> 32));
    }
    uint32_t Q[NL];
    uint64_t rem = 0;
    for (int i = NL - 1; i >= 0; --i) {
      const uint64_t cur = (rem << 32) | L[i];
      Q[i] = static_cast<uint32_t>(cur / d);
      rem = cur % d;
    }
    int h = -1;
    for (int i = NL - 1; i >= 0 && h < 0; --i)
      if (Q[i]) h = i * 32 + 31 - __clz(Q[i]);
    if (h < 23) {
      const uint32_t q = Q[0];
      const bool up = (2 * rem > d) || (2 * rem == d && (q & 1u));
      bits = q + (up ? 1u : 0u);
    } else {
      const int shift = h - 23;
      uint32_t mant = 0;
      for (int b = 0; b < 24; ++b) mant |= static_cast<uint32_t>(bit_of(Q, shift + b)) << b;
      bool up;
      if (shift == 0) {
        up = (2 * rem > d) || (2 * rem == d && (mant & 1u));
      } else {
        const int rb = bit_of(Q, shift - 1);
        bool sticky = rem != 0;
        for (int b = 0; b < shift - 1 && !sticky; ++b) sticky = bit_of(Q, b);
        up = rb && (sticky || (mant & 1u));
      }
      mant += up ? 1u : 0u;
      bits = (static_cast<uint32_t>(shift + 1) << 23) + (mant - 0x800000u);
    }
  }
  *offset = __uint_as_float(bits);
}

// One CTA of 256 threads per group of 256 centred scales.  The 255 distinct
// codebook values V_0 < ... < V_254 are: -|T|(127..1), 0, |T|(1..127); the
// code of the nearest value to c/s2 (ties to the smaller value) is the number
// k of midpoints (V_k + V_{k+1})/2 with s2 * mid < c, decided in fp64 where
// s2 * mid is exact; k < 127 -> byte 0x80 | (127 - k), k = 127 -> 0x00,
// k > 127 -> byte k - 127.
__global__ void __launch_bounds__(256) dq_encode_kernel(const float* __restrict__ a, int64_t n1,
                                                        const float* __restrict__ offset_p,
                                                        uint8_t* __restrict__ code8,
                                                        float* __restrict__ s2) {
  __shared__ float mag[128];
  __shared__ double mid[254];
  __shared__ float wmax[8];
  for (int t = threadIdx.x; t < 128; t += blockDim.x) mag[t] = t8_magnitude(t);
  __syncthreads();
  for (int k = threadIdx.x; k < 254; k += blockDim.x) {
    auto V = [&](int i) -> double {
      return i < 127 ? -static_cast<double>(mag[127 - i])
                     : (i == 127 ? 0.0 : static_cast<double>(mag[i - 127]));
    };
    mid[k] = 0.5 * (V(k) + V(k + 1));
  }
  const int64_t g = blockIdx.x;
  const int64_t i = g * kDQBlock + threadIdx.x;
  const float off = *offset_p;
  const bool valid = i < n1;
  const float c = valid ? __fsub_rn(a[i], off) : 0.0f;
  float m = fabsf(c);
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  float sg = wmax[0];
  for (int w = 1; w < 8; ++w) sg = fmaxf(sg, wmax[w]);
  if (!(sg > 0.0f)) sg = 1.0f;
  if (threadIdx.x == 0) s2[g] = sg;
  if (!valid) return;
  const double cd = static_cast<double>(c), sd = static_cast<double>(sg);
  int lo = 0, hi = 254;  // find the first k with sd*mid[k] >= cd
  while (lo < hi) {
    const int md = (lo + hi) >> 1;
    if (sd * mid[md] < cd)
      lo = md + 1;
    else
      hi = md;
  }
  const int k = lo;
  const uint32_t byte = k < 127 ? (0x80u | static_cast<uint32_t>(127 - k))
                                : (k == 127 ? 0u : static_cast<uint32_t>(k - 127));
  code8[i] = static_cast<uint8_t>(byte);
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
cudaError_t launch_quantize(const void* W, int dtype, int64_t numel, uint8_t* packed,
                            float* absmax_out, bool dq, uint8_t* code8, float* s2, float* offset,
                            void* ws, int32_t* d_status, cudaStream_t st, int num_sms) {
  const int64_t n1 = (numel + kBlock - 1) / kBlock;
  const int threads = 256;
  const int64_t want = (n1 * 8 + threads - 1) / threads;
  const int blocks = static_cast<int>(want < num_sms * 8LL ? want : num_sms * 8LL);
  unsigned long long* bins = nullptr;
  float* scales = absmax_out;
  if (dq) {
    bins = static_cast<unsigned long long*>(ws);
    scales = reinterpret_cast<float*>(static_cast<char*>(ws) + 2048);
    cudaError_t e = cudaMemsetAsync(bins, 0, 2048, st);
    if (e != cudaSuccess) return e;
  }
  {
  ProfScope prof(kProfQuantize, st);
  if (dtype == QLORA_DTYPE_BF16) {
    if (dq)
      nf4_encode_kernel<uint16_t, true><<<blocks, threads, 0, st>>>(
          static_cast<const uint16_t*>(W), numel, n1, packed, scales, bins, d_status);
    else
      nf4_encode_kernel<uint16_t, false><<<blocks, threads, 0, st>>>(
          static_cast<const uint16_t*>(W), numel, n1, packed, scales, bins, d_status);
  } else {
    if (dq)
      nf4_encode_kernel<float, true><<<blocks, threads, 0, st>>>(
          static_cast<const float*>(W), numel, n1, packed, scales, bins, d_status);
    else
      nf4_encode_kernel<float, false><<<blocks, threads, 0, st>>>(
          static_cast<const float*>(W), numel, n1, packed, scales, bins, d_status);
  }
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || !dq) return e;
  {
    ProfScope prof(kProfQuantize, st);
    dq_mean_kernel<<<1, 256, 0, st>>>(bins, n1, offset);
  }
  const int64_t n2 = (n1 + kDQBlock - 1) / kDQBlock;
  {
    ProfScope prof(kProfQuantize, st);
    dq_encode_kernel<<<static_cast<unsigned>(n2), 256, 0, st>>>(scales, n1, offset, code8, s2);
  }
  return cudaGetLastError();
}

size_t quantize_workspace_bytes(int64_t numel, bool dq) {
  if (!dq) return 0;
  const int64_t n1 = (numel + kBlock - 1) / kBlock;
  return 2048 + static_cast<size_t>(n1) * 4;
}

}  // namespace qnf4
