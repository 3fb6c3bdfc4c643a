// NF4 encoder (absmax, nearest code, nibble pack) and double quantization of
// the block scales.  Page "QLoRA：冻结的 4-bit 权重怎样参与一次微调",
// §NF4 保存的是索引而不是均匀整数值, §从 NF4 索引打包成字节,
// §Double Quantization 压缩的是 Scale.
#include <atomic>
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
// The fast path computes t = w * (1/s) in fp32 (absolute error < 2^-21) and
// looks t up in 33 uniform buckets of width 1/16 that are offset by half a
// bucket; every bucket holds at most one midpoint and no midpoint lies within
// 0.004 of a bucket edge, so a bucket gives (number of midpoints below it,
// the midpoint inside it).  A bucket's entry is one 32-bit word: the fp32
// midpoint (4.0 when the bucket holds none) with its low five mantissa bits
// replaced by (number of midpoints below the bucket) + 1.  That moves the
// midpoint by under 32 ulp, i.e. under 2^-19 since |m| < 1; with the 2^-21
// error of t the computed t - m is within E < 2^-18 of the exact one, so its
// sign can be wrong only when |t - m| < 2E < 2^-17.  Every element within
// 2^-17 of the stored midpoint (exact ties included) is therefore redone
// exactly: w > s*m_j in fp64, where s*m_j is exact (24-bit times at most
// 26-bit significand).  An exact tie (w == s*m_j) is not "greater", so it
// keeps the smaller index.  Each lane reads its own copy of the 33 words
// (bucket b of lane l at word 32b + l), so the lookups of a warp never
// conflict.
// ---------------------------------------------------------------------------
constexpr int kBuckets = 33;
constexpr float kNearEps = 7.62939453125e-06f;   // 2^-17

// The buckets, formed at compile time: bucket b covers t in
// [(b - 16.5)/16, (b - 15.5)/16); mid = the fp32 midpoint inside it (4.0 when
// none), below = number of midpoints below it + 1; and the 15 midpoints in fp64.
struct BucketTables {
  float mid[kBuckets];
  uint32_t below[kBuckets];
  double mexact[15];
};

constexpr float kNF4host[16] = {QNF4_TABLE_VALUES};

constexpr BucketTables make_bucket_tables() {
  BucketTables t{};
  for (int b = 0; b < kBuckets; ++b) {
    const double lo = (b - 16.5) / 16.0, hi = (b - 15.5) / 16.0;
    int jlo = 0;
    float mid = 4.0f;
    for (int j = 0; j < 15; ++j) {
      const double mj = 0.5 * (static_cast<double>(kNF4host[j]) + static_cast<double>(kNF4host[j + 1]));
      if (mj < lo)
        ++jlo;
      else if (mj < hi)
        mid = static_cast<float>(mj);
    }
    t.mid[b] = mid;
    t.below[b] = static_cast<uint32_t>(jlo + 1);
  }
  for (int j = 0; j < 15; ++j)
    t.mexact[j] = 0.5 * (static_cast<double>(kNF4host[j]) + static_cast<double>(kNF4host[j + 1]));
  return t;
}
static_assert(make_bucket_tables().below[0] == 1 && make_bucket_tables().below[kBuckets - 1] == 16 &&
                  make_bucket_tables().mid[16] == 4.0f,
              "bucket table spot values");

static __constant__ BucketTables kBucketTab = make_bucket_tables();

// Per-lane copies of the bucket entries in shared memory (entry b of lane l at
// index 32b + l; the 32 threads of a warp read one constant word at a time):
// tab4 holds the midpoint with its low five bits replaced by `below`, tab8 the
// pair (midpoint, below); either may be null.
__device__ __forceinline__ void load_buckets(uint32_t* tab4, uint2* tab8, double* mexact) {
  for (int i = threadIdx.x; i < kBuckets * 32; i += blockDim.x) {
    const int b = i >> 5;
    const uint32_t m = __float_as_uint(kBucketTab.mid[b]), j1 = kBucketTab.below[b];
    if (tab4 != nullptr) tab4[i] = (m & ~31u) | j1;
    if (tab8 != nullptr) tab8[i] = make_uint2(m, j1);
  }
  for (int j = threadIdx.x; j < 15; j += blockDim.x) mexact[j] = kBucketTab.mexact[j];
}

__device__ __forceinline__ void build_buckets(uint32_t* tab /*[33][32]*/, double* mexact) {
  load_buckets(tab, nullptr, mexact);
}

// Exact decision for one element: code = jlo + (x > s*m_jlo) with the product
// exact in fp64 (x, s already scaled alike).
__device__ __forceinline__ uint32_t exact_code(float x, float s, int jlo, const double* mexact) {
  return static_cast<uint32_t>(jlo) +
         (static_cast<double>(x) > static_cast<double>(s) * mexact[jlo] ? 1u : 0u);
}

constexpr int kLaneElems = 16;   // consecutive elements per lane; 4 lanes per 64-block

template <typename T>
__device__ __forceinline__ void load16(const T* __restrict__ W, int64_t e0, int64_t numel,
                                       bool fast, float (&x)[kLaneElems]);

template <>
__device__ __forceinline__ void load16<uint16_t>(const uint16_t* __restrict__ W, int64_t e0,
                                                 int64_t numel, bool fast,
                                                 float (&x)[kLaneElems]) {
  if (fast) {
    const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(W + e0));
    const uint4 v1 = __ldg(reinterpret_cast<const uint4*>(W + e0 + 8));
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int i = 0; i < kLaneElems; ++i)
      x[i] = (e0 + i < numel) ? bf16_bits_to_f32(__ldg(W + e0 + i)) : 0.0f;
  }
}

template <>
__device__ __forceinline__ void load16<float>(const float* __restrict__ W, int64_t e0,
                                              int64_t numel, bool fast, float (&x)[kLaneElems]) {
  if (fast) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(W + e0 + 4 * i));
      x[4 * i] = v.x; x[4 * i + 1] = v.y; x[4 * i + 2] = v.z; x[4 * i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < kLaneElems; ++i) x[i] = (e0 + i < numel) ? __ldg(W + e0 + i) : 0.0f;
  }
}

// Per block-leader lane: the scales' exact sum per exponent is kept in two
// (exponent, sum) register slots and only flushed to the CTA's shared bins
// when a third exponent shows up, so the bins see few atomics.
struct BinCache {
  uint32_t k0 = 0, k1 = 0;
  unsigned long long s0 = 0, s1 = 0;
  __device__ __forceinline__ void add(float scale, unsigned long long* sbins) {
    const uint32_t u = __float_as_uint(scale);
    const uint32_t E = (u >> 23) & 0xFFu;
    const uint32_t mant = (u & 0x7FFFFFu) | (E ? 0x800000u : 0u);
    const uint32_t key = E ? E : 1u;
    if (key == k0) {
      s0 += mant;
    } else if (key == k1) {
      s1 += mant;
    } else {
      if (s1) atomicAdd(&sbins[k1], s1);
      k1 = k0;
      s1 = s0;
      k0 = key;
      s0 = mant;
    }
  }
  __device__ __forceinline__ void flush(unsigned long long* sbins) {
    if (s0) atomicAdd(&sbins[k0], s0);
    if (s1) atomicAdd(&sbins[k1], s1);
  }
};

// Encode the 16 elements x[] of one lane (lane `sub` of its 4-lane group,
// elements e0..e0+15 of 64-block blk): absmax over the group, nearest codes,
// packed store; the group leader stores the scale.
//
// Per element the fast path is: t = x/s by one multiply with an approximate
// reciprocal; bucket = round(16 t + 16) by adding 2^23 + 16 (exact integer in
// the low mantissa bits, no conversion instruction); one shared load of
// (midpoint, codes below it); code = codes below + (t > midpoint) from the
// sign of t - midpoint.  Exact fp64 decisions redo the rare elements within
// 2^-20 of their midpoint (which includes t equal to it).
template <bool kDQ>
__device__ __forceinline__ void encode16(float (&x)[kLaneElems], int64_t blk, int64_t e0, int sub,
                                         unsigned gmask, int64_t numel, bool full,
                                         const uint32_t* tab, const double* mexact,
                                         uint8_t* __restrict__ packed, float* __restrict__ scales,
                                         BinCache& bc, unsigned long long* sbins, bool& bad) {
  float am = 0.0f;
#pragma unroll
  for (int i = 0; i < kLaneElems; ++i) am = fmax_nan(am, fabsf(x[i]));
  am = fmax_nan(am, __shfl_xor_sync(gmask, am, 1));
  am = fmax_nan(am, __shfl_xor_sync(gmask, am, 2));
  const bool finite = am <= FLT_MAX;
  bad |= !finite;
  const float s = (finite && am > 0.0f) ? am : 1.0f;
  uint32_t w0 = 0x77777777u, w1 = 0x77777777u;   // all code 7 (non-finite blocks, padding)
  if (finite) {
    // Keep s and 1/s normal: a block scale below 2^-126 (1/s would overflow)
    // is scaled up by 2^64, one above 2^126 (1/s would be subnormal) down by
    // 2^-64, together with its elements; codes depend only on w/s, and an
    // element that loses bits this way is far below any midpoint.
    float s_eff = s;
    if (s < 1.17549435e-38f || s > 8.50705917e37f) {
      const float sc = s < 1.17549435e-38f ? 18446744073709551616.0f : 5.42101086e-20f;
#pragma unroll
      for (int i = 0; i < kLaneElems; ++i) x[i] *= sc;
      s_eff = s * sc;
    }
    // relative error of t below 2^-21 (inside the exact check's window, above)
    float inv_s;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(inv_s) : "f"(s_eff));
    // (bits of 2^23 + b) * 128 + tb = this lane's word of bucket b
    const uint32_t tb = smem_u32(tab) + (threadIdx.x & 31u) * 4u - 0x4B000000u * 128u;
    float dmin = 1.0f;
    w0 = 0;
    w1 = 0;
#pragma unroll
    for (int i = 0; i < kLaneElems; ++i) {
      const float t = x[i] * inv_s;
      const float y = fmaf(t, 16.0f, 8388624.0f);             // 2^23 + 16 + 16 t, rounded to an integer
      uint32_t ent;
      asm("ld.shared.b32 %0, [%1];" : "=r"(ent) : "r"(tb + __float_as_uint(y) * 128u));
      const float d = t - __uint_as_float(ent);
      // codes below the bucket + 1, minus one when t is below the midpoint
      const uint32_t code = (ent & 31u) - (__float_as_uint(d) >> 31);
      dmin = fminf(dmin, fabsf(d));
      const int sh = (i & 7) >> 1;
      if (i < 8)
        w0 += code << (sh * 8 + ((i & 1) ? 0 : 4));
      else
        w1 += code << (sh * 8 + ((i & 1) ? 0 : 4));
    }
    if (dmin < kNearEps) {
      w0 = 0;
      w1 = 0;
#pragma unroll
      for (int i = 0; i < kLaneElems; ++i) {
        const float t = x[i] * inv_s;
        const int b = __float2int_rd(fmaf(t, 16.0f, 16.5f));
        const uint32_t ent = tab[32 * (b < 0 ? 0 : (b > kBuckets - 1 ? kBuckets - 1 : b))];
        const int jlo = static_cast<int>(ent & 31u) - 1;
        const float d = t - __uint_as_float(ent);
        uint32_t code = static_cast<uint32_t>(jlo) + (d > 0.0f ? 1u : 0u);
        if (fabsf(d) < kNearEps) code = exact_code(x[i], s_eff, jlo, mexact);
        const int sh = (i & 7) >> 1;
        if (i < 8)
          w0 += code << (sh * 8 + ((i & 1) ? 0 : 4));
        else
          w1 += code << (sh * 8 + ((i & 1) ? 0 : 4));
      }
    }
    if (!full) {
#pragma unroll
      for (int i = 0; i < kLaneElems; ++i)
        if (e0 + i >= numel) {
          const int sh = ((i & 7) >> 1) * 8 + ((i & 1) ? 0 : 4);
          uint32_t& w = i < 8 ? w0 : w1;
          w = (w & ~(0xFu << sh)) | (static_cast<uint32_t>(kPadCode) << sh);
        }
    }
  }
  const int64_t b0 = e0 >> 1;
  if (full) {
    *reinterpret_cast<uint2*>(packed + b0) = make_uint2(w0, w1);
  } else {
    const int64_t nbytes = (numel + 1) >> 1;
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (b0 + k < nbytes) packed[b0 + k] = static_cast<uint8_t>((k < 4 ? w0 : w1) >> (8 * (k & 3)));
  }
  if (sub == 0) {
    scales[blk] = s;
    if (kDQ) bc.add(s, sbins);
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
// Exact mean of the n1 first-level scales from their exponent bins: the
// range of non-empty keys (warp 0, ballots) ...
__device__ __forceinline__ void bins_key_range(const unsigned long long* sb, int* range) {
  if (threadIdx.x < 32) {
    uint32_t m = 0;
    for (int i = 0; i < 8; ++i) m |= (sb[threadIdx.x * 8 + i] != 0ull ? 1u : 0u) << i;
    const unsigned any = __ballot_sync(0xFFFFFFFFu, m != 0);
    if (any == 0u) {
      // no scale was binned (shards that covered no block): an empty range,
      // which exact_mean_bits turns into a mean of 0
      if (threadIdx.x == 0) {
        range[0] = 1;
        range[1] = 0;
      }
      return;
    }
    const int lmin = __ffs(any) - 1, lmax = 31 - __clz(any);
    if (threadIdx.x == lmin) range[0] = threadIdx.x * 8 + (__ffs(m) - 1);
    if (threadIdx.x == lmax) range[1] = threadIdx.x * 8 + (31 - __clz(m));
  }
}

// floor(S / d) and S mod d for S < 2^126 and 0 < d < 2^62, without a
// bit-serial division: three rounds of (double-precision quotient of the
// remaining remainder, exact 128-bit correction of quotient and remainder);
// each round shrinks the remainder by about 2^50, so the third leaves it
// within one divisor of the final range, which the last steps settle exactly.
__device__ __forceinline__ double u128_to_f64(unsigned __int128 v) {
  return static_cast<double>(static_cast<uint64_t>(v >> 64)) * 18446744073709551616.0 +
         static_cast<double>(static_cast<uint64_t>(v));
}

__device__ __forceinline__ unsigned __int128 f64_to_u128(double v) {   // v >= 0, < 2^127
  const double hi = floor(v * 5.421010862427522e-20);                 // v / 2^64
  const double lo = v - hi * 18446744073709551616.0;                    // exact
  return (static_cast<unsigned __int128>(static_cast<uint64_t>(hi)) << 64) +
         static_cast<unsigned __int128>(static_cast<uint64_t>(lo));
}

__device__ void divmod_u128_u64(unsigned __int128 S, uint64_t d, unsigned __int128& Q, uint64_t& R) {
  const double dd = static_cast<double>(d);
  unsigned __int128 q = 0;
  __int128 r = static_cast<__int128>(S);
  for (int round = 0; round < 3; ++round) {
    const bool neg = r < 0;
    const unsigned __int128 adj =
        f64_to_u128(floor(u128_to_f64(static_cast<unsigned __int128>(neg ? -r : r)) / dd));
    if (neg) {
      q -= adj;
      r += static_cast<__int128>(adj * d);
    } else {
      q += adj;
      r -= static_cast<__int128>(adj * d);
    }
  }
  for (int i = 0; i < 4 && r < 0; ++i) {
    --q;
    r += d;
  }
  for (int i = 0; i < 4 && r >= static_cast<__int128>(d); ++i) {
    ++q;
    r -= d;
  }
  Q = q;
  R = static_cast<uint64_t>(r);
}

// ... and the sum divided by n1 with one rounding to fp32 (one thread).
__device__ uint32_t exact_mean_bits(const unsigned long long* sb, int kmin, int kmax, int64_t n1) {
  const uint64_t d = static_cast<uint64_t>(n1);
  uint32_t bits;
  if (kmax - kmin <= 64) {
    unsigned __int128 S = 0;
    for (int key = kmin; key <= kmax; ++key)
      S += static_cast<unsigned __int128>(sb[key]) << (key - kmin);
    unsigned __int128 Q;
    uint64_t rem;
    if ((S >> 126) == 0 && (d >> 62) == 0) {
      divmod_u128_u64(S, d, Q, rem);
    } else {
      Q = S / d;
      rem = static_cast<uint64_t>(S % d);
    }
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
  return bits;
}

constexpr int kChunkBlocks = 64;                 // 64-blocks per streamed chunk
constexpr int kChunkElems = kChunkBlocks * kBlock;
constexpr int kEncStages = 4;

template <typename T>
constexpr size_t encode_smem_bytes() {
  return static_cast<size_t>(kEncStages) * kChunkElems * sizeof(T) + 128;
}

// CTA = 256 threads = 64 groups of 4 lanes = one chunk of 64 blocks per
// iteration.  Whole chunks stream into a 4-stage shared-memory ring by 1-D
// bulk copies; the remaining blocks (a partial last chunk, or everything when
// W is not 16-byte aligned) are read directly from global memory.
//
// The workspace head (exponent bins, finished-CTA counter) is cleared by CTA 0
// at the start of every call, which then publishes the call's token; every
// CTA waits for that token before adding its bins (at its end, long after),
// so no separate clearing step has to run before the kernel.
__device__ __forceinline__ unsigned long long* ws_token(unsigned long long* bins) {
  return reinterpret_cast<unsigned long long*>(reinterpret_cast<char*>(bins) + 2056);
}

// The claimed-chunk counter of the bf16 encoder (chunks past its first waves).
__device__ __forceinline__ unsigned long long* ws_chunk_counter(unsigned long long* bins) {
  return reinterpret_cast<unsigned long long*>(reinterpret_cast<char*>(bins) + 2072);
}

__device__ __forceinline__ void ws_clear_and_publish(unsigned long long* bins, unsigned int* done_ctas,
                                                     unsigned long long token) {
  if (blockIdx.x != 0) return;
  for (int i = threadIdx.x; i < 256; i += blockDim.x) bins[i] = 0ull;
  if (threadIdx.x == 0 && done_ctas != nullptr) *done_ctas = 0u;
  if (threadIdx.x == 0) *ws_chunk_counter(bins) = 0ull;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(ws_token(bins)), "l"(token) : "memory");
  }
}

// true once CTA 0 has cleared the head for this call (bounded wait)
__device__ __forceinline__ bool ws_wait_published(unsigned long long* bins, unsigned long long token) {
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(ws_token(bins)) : "memory");
    if (v == token) return true;
    if (globaltimer_ns() - t0 > 2000000000ull) return false;
    __nanosleep(64);
  }
}

// The call's token again once the last CTA has stored the mean (the encoder
// that also double-quantizes in the same launch).
__device__ __forceinline__ unsigned long long* ws_mean_flag(unsigned long long* bins) {
  return reinterpret_cast<unsigned long long*>(reinterpret_cast<char*>(bins) + 2064);
}

__device__ __forceinline__ bool ws_wait_mean(unsigned long long* bins, unsigned long long token) {
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(ws_mean_flag(bins)) : "memory");
    if (v == token) return true;
    if (globaltimer_ns() - t0 > 2000000000ull) return false;
    __nanosleep(128);
  }
}

template <typename T, bool kDQ>
__global__ void __launch_bounds__(256) nf4_encode_kernel(const T* __restrict__ W, int64_t numel,
                                                         int64_t n1, uint8_t* __restrict__ packed,
                                                         float* __restrict__ scales,
                                                         unsigned long long* __restrict__ bins,
                                                         unsigned int* __restrict__ done_ctas,
                                                         float* __restrict__ offset_out,
                                                         int32_t* d_status, unsigned long long token) {
  extern __shared__ uint8_t esm_raw[];
  T* ring = reinterpret_cast<T*>((reinterpret_cast<uintptr_t>(esm_raw) + 127) &
                                 ~static_cast<uintptr_t>(127));
  __shared__ uint32_t tab[kBuckets * 32];
  __shared__ double mexact[15];
  __shared__ unsigned long long sbins[kDQ ? 256 : 1];
  __shared__ uint64_t full_bar[kEncStages];
  pdl_launch_dependents();
  pdl_wait();
  if (kDQ) ws_clear_and_publish(bins, done_ctas, token);
  __shared__ int abort_flag;
  build_buckets(tab, mexact);
  if (kDQ)
    for (int i = threadIdx.x; i < 256; i += blockDim.x) sbins[i] = 0ull;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kEncStages; ++i) mbar_init(&full_bar[i], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int sub = lane & 3;
  const unsigned gmask = 0xFu << (lane & 28);
  const bool aligned16 = (reinterpret_cast<uintptr_t>(W) & 15u) == 0;
  const int64_t nchunks = aligned16 ? numel / kChunkElems : 0;
  const int64_t my_n =
      nchunks > blockIdx.x ? (nchunks - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  constexpr uint32_t kChunkBytes = kChunkElems * sizeof(T);
  BinCache bc;
  bool bad = false;

  if (threadIdx.x == 0) {
    for (int64_t j = 0; j < my_n && j < kEncStages; ++j) {
      const int64_t c = blockIdx.x + j * gridDim.x;
      mbar_arrive_expect_tx(&full_bar[j], kChunkBytes);
      bulk_load_1d(ring + j * kChunkElems, W + c * kChunkElems, kChunkBytes, &full_bar[j]);
    }
  }
  for (int64_t j = 0; j < my_n; ++j) {
    const int s = static_cast<int>(j % kEncStages);
    const uint32_t ph = static_cast<uint32_t>((j / kEncStages) & 1);
    if (!mbar_wait(&full_bar[s], ph)) abort_flag = 1;
    __syncthreads();
    if (abort_flag) break;
    const int64_t c = blockIdx.x + j * gridDim.x;
    const int local = threadIdx.x >> 2;
    const int64_t blk = c * kChunkBlocks + local;
    const int64_t e0 = blk * kBlock + sub * kLaneElems;
    const T* src = ring + s * kChunkElems + local * kBlock + sub * kLaneElems;
    float x[kLaneElems];
    if (sizeof(T) == 2) {
      const uint4 v0 = *reinterpret_cast<const uint4*>(src);
      const uint4 v1 = *reinterpret_cast<const uint4*>(src + 8);
      const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 v = *reinterpret_cast<const float4*>(src + 4 * i);
        x[4 * i] = v.x; x[4 * i + 1] = v.y; x[4 * i + 2] = v.z; x[4 * i + 3] = v.w;
      }
    }
    __syncthreads();   // every thread has its values: the stage may be refilled
    if (threadIdx.x == 0 && j + kEncStages < my_n) {
      const int64_t c2 = blockIdx.x + (j + kEncStages) * gridDim.x;
      mbar_arrive_expect_tx(&full_bar[s], kChunkBytes);
      bulk_load_1d(ring + s * kChunkElems, W + c2 * kChunkElems, kChunkBytes, &full_bar[s]);
    }
    encode16<kDQ>(x, blk, e0, sub, gmask, numel, true, tab, mexact, packed, scales, bc, sbins, bad);
  }
  if (abort_flag && threadIdx.x == 0) raise_status(d_status, QLORA_ERR_TIMEOUT);
  // blocks not covered by whole streamed chunks
  const int64_t first = nchunks * kChunkBlocks;
  const int64_t ngroups = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 2;
  for (int64_t blk = first + ((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 2);
       blk < n1; blk += ngroups) {
    const int64_t e0 = blk * kBlock + sub * kLaneElems;
    const bool full = e0 + kLaneElems <= numel;
    float x[kLaneElems];
    load16<T>(W, e0, numel, full && aligned16, x);
    encode16<kDQ>(x, blk, e0, sub, gmask, numel, full, tab, mexact, packed, scales, bc, sbins, bad);
  }
  if (bad) raise_status(d_status, QLORA_ERR_NONFINITE);
  if (kDQ) {
    if (sub == 0) bc.flush(sbins);
    __shared__ int published;
    if (threadIdx.x == 0) {
      published = ws_wait_published(bins, token) ? 1 : 0;
      if (!published) raise_status(d_status, QLORA_ERR_TIMEOUT);
    }
    __syncthreads();
    if (published)
      for (int i = threadIdx.x; i < 256; i += blockDim.x)
        if (sbins[i]) atomicAdd(&bins[i], sbins[i]);
    // The last CTA to finish forms the exact mean of all first-level scales
    // from the global bins (every other CTA's additions are visible to it:
    // each made them before its fenced increment of the counter).
    __shared__ int last_cta;
    __shared__ int krange[2];
    __syncthreads();
    if (offset_out == nullptr) return;   // a shard: the caller adds the bins of all shards
    if (threadIdx.x == 0) {
      __threadfence();
      last_cta = atomicAdd(done_ctas, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (last_cta) {
      __threadfence();
      for (int i = threadIdx.x; i < 256; i += blockDim.x) sbins[i] = __ldcg(bins + i);
      __syncthreads();
      bins_key_range(sbins, krange);
      __syncthreads();
      if (threadIdx.x == 0) *offset_out = __uint_as_float(exact_mean_bits(sbins, krange[0], krange[1], n1));
    }
  }
}

// ---------------------------------------------------------------------------
// Double quantization of the scales: groups of 256 centred scales, one warp
// per group.  The 255 distinct codebook values V_0 < ... < V_254 are: -|T|(127..1), 0,
// |T|(1..127); the code of the nearest value to c/s2 (ties to the smaller
// value) is the number k of midpoints m_k = (V_k + V_{k+1})/2 with
// s2 * m_k < c.  s2 * m_k is exact in fp64, and for an fp32 c,
// c > s2 * m_k  <=>  c > RD_fp32(s2 * m_k); so each warp turns its group's
// 254 midpoints into fp32 thresholds T once, and the count k comes from a
// cell table (below) and one comparison with T.
// k < 127 -> byte 0x80 | (127 - k), k = 127 -> 0x00, k > 127 -> byte k - 127.
// The 254 midpoints between consecutive values of the sorted 255-value
// codebook V (-|T|(127..1), 0, |T|(1..127)), in fp64, formed at compile time.
struct T8Midpoints {
  double m[254];
};

constexpr T8Midpoints make_t8_midpoints() {
  T8Midpoints r{};
  const T8Table t = make_t8_table();
  auto V = [&t](int i) -> double {
    return i < 127 ? -static_cast<double>(t.v[127 - i])
                   : (i == 127 ? 0.0 : static_cast<double>(t.v[i - 127]));
  };
  for (int k = 0; k < 254; ++k) r.m[k] = 0.5 * (V(k) + V(k + 1));
  return r;
}

// Cells of x = c / s2 (as the fp32 product c * RN(1/s2), within 2^-23 of the
// exact quotient, relative): the sign, the binade 2^-21 .. 2^0 (row 1 .. 22;
// row 0 = |x| < 2^-21, below the smallest nonzero midpoint 5e-7) and the top
// 6 mantissa bits (64 cells per row).  Widened by 2^-20 (relative) on both
// sides, every cell holds at most one midpoint (checked at compile time: the
// smallest gap between positive midpoints is 1.4%).  Entry k0 = the number of
// midpoints certainly below any x of the cell, so the exact count is k0, or
// k0 + 1 when T[k0] < c.  Positive cells follow the 127 negative midpoints;
// negative cells count, by symmetry (m_{253-i} = -m_i), the midpoints above
// -x.
constexpr int kT8Rows = 23;
constexpr int kT8CellBits = 6;
constexpr int kT8SignCells = kT8Rows << kT8CellBits;   // cells per sign

struct alignas(16) T8Cells {
  uint8_t k0[2 * kT8SignCells];   // [0, kT8SignCells): x >= 0; then x < 0
  int most_per_cell;              // compile-time check of the one-midpoint rule
};

constexpr T8Cells make_t8_cells() {
  T8Cells r{};
  const T8Midpoints mp = make_t8_midpoints();
  const double widen = 1.0 / 1048576.0;   // 2^-20
  int below = 0, upto = 0;                // positive midpoints < lo', <= hi'
  r.most_per_cell = 0;
  for (int row = 0; row < kT8Rows; ++row) {
    double p2 = 1.0;                      // 2^(row - 22): the row's binade
    for (int i = row; i < kT8Rows - 1; ++i) p2 *= 0.5;
    for (int cell = 0; cell < (1 << kT8CellBits); ++cell) {
      // row 0 (every cell alike): 0 <= |x| < 2^-21
      const double lo = row == 0 ? 0.0 : p2 * (1.0 + cell / 64.0);
      const double hi = row == 0 ? 2.0 * p2 : p2 * (1.0 + (cell + 1) / 64.0);
      while (below < 127 && mp.m[127 + below] < lo * (1.0 - widen)) ++below;
      while (upto < 127 && mp.m[127 + upto] <= hi * (1.0 + widen)) ++upto;
      const int idx = (row << kT8CellBits) + cell;
      r.k0[idx] = static_cast<uint8_t>(127 + below);
      r.k0[kT8SignCells + idx] = static_cast<uint8_t>(127 - upto);
      if (upto - below > r.most_per_cell) r.most_per_cell = upto - below;
    }
  }
  return r;
}
static_assert(make_t8_cells().most_per_cell <= 1, "a T8 cell holds more than one midpoint");

// global (not constant) memory: each thread of a CTA reads a different entry
static __device__ const T8Midpoints kT8Mid = make_t8_midpoints();
static __device__ const T8Cells kT8Cells = make_t8_cells();

// The count of thresholds s2 * m_k below c by binary search (sd = s2, in
// fp64, where each product is exact); the path of groups whose 1/s2 is not a
// normal number.
__device__ __noinline__ int t8_search(double cd, double sd, const double* mid) {
  int lo = 0, hi = 254;
#pragma unroll 1
  for (int it = 0; it < 8; ++it) {
    const int md = min((lo + hi) >> 1, 253);   // < 254 whenever lo < hi
    const bool less = sd * mid[md] < cd;
    lo = (lo < hi && less) ? md + 1 : lo;
    hi = (lo < hi && !less) ? md : hi;
  }
  return lo;
}

// The code byte of one centred scale c (see above): x = c * inv_s2, its
// cell's k0 from the table `cells` and one comparison of c with the exact
// threshold s2 * m_{k0} in fp64 (sd = s2).  |x| >= 2 or not finite (inv_s2 =
// infinity: see the caller) takes a binary search over the thresholds
// instead.  Index k -> byte: k >= 127 -> k - 127, k < 127 -> 0x80 | (127 - k).
__device__ __forceinline__ uint32_t t8_code_byte(float c, float inv_s2, double sd,
                                                 const uint8_t* cells, const double* mid) {
  const uint32_t xb = __float_as_uint(c * inv_s2);
  const double cd = static_cast<double>(c);
  // cells are (|x| bits >> 17) - (105 << 6): row 0 holds every |x| < 2^-21
  const int r = max(static_cast<int>((xb & 0x7FFFFFFFu) >> 17) - (105 << kT8CellBits), 0);
  int k;
  if (r >= kT8SignCells) {
    k = t8_search(cd, sd, mid);
  } else {
    const int k0 = cells[static_cast<int>(xb >> 31) * kT8SignCells + r];
    k = k0 + ((k0 < 254 && sd * mid[min(k0, 253)] < cd) ? 1 : 0);
  }
  return static_cast<uint32_t>(k >= 127 ? k - 127 : 255 - k);
}

// Second-level scale and scale codes of group g (one warp; lane l holds
// scales 4l..4l+3 and 128+4l..128+4l+3 of the group): c = a - offset,
// s2 = max |c| (1 for an all-zero group), then each code from the cell table
// and one threshold.  The scales are read through L2 (ld.global.cg): in the
// encoder's own launch other CTAs wrote them.  `a` is 16-byte aligned.
__device__ __forceinline__ void dq_encode_group(const float* a, int64_t n1, int64_t g, float off,
                                                const double* mid, const uint8_t* cells,
                                                uint8_t* __restrict__ code8, float* __restrict__ s2,
                                                int lane) {
  const int64_t base = g * kDQBlock;
  const bool whole = base + kDQBlock <= n1;
  float c[8];
  if (whole) {
    const float4 v0 = __ldcg(reinterpret_cast<const float4*>(a + base) + lane);
    const float4 v1 = __ldcg(reinterpret_cast<const float4*>(a + base + 128) + lane);
    c[0] = v0.x; c[1] = v0.y; c[2] = v0.z; c[3] = v0.w;
    c[4] = v1.x; c[5] = v1.y; c[6] = v1.z; c[7] = v1.w;
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t i = base + (j >> 2) * 128 + 4 * lane + (j & 3);
      c[j] = i < n1 ? __ldcg(a + i) : off;   // past the end: c = 0
    }
  }
  float m = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    c[j] = __fsub_rn(c[j], off);
    m = fmaxf(m, fabsf(c[j]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  const float sg = m > 0.0f ? m : 1.0f;
  if (lane == 0) s2[g] = sg;
  const double sd = static_cast<double>(sg);
  // 1/s2 within 2^-24 (relative) while it is a normal number; outside
  // 2^-128 <= s2 < 2^126 the group searches the thresholds instead (infinity)
  const float inv_s2 = (sg >= 2.938735877e-39f && sg < 8.507059173e37f)
                           ? 1.0f / sg : __int_as_float(0x7F800000);
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int j = 0; j < 8; ++j)
    w[j >> 2] |= t8_code_byte(c[j], inv_s2, sd, cells, mid) << (8 * (j & 3));
  uint8_t* dst = code8 + base + 4 * lane;
  if (whole && (reinterpret_cast<uintptr_t>(code8 + base) & 3u) == 0) {
    *reinterpret_cast<uint32_t*>(dst) = w[0];
    *reinterpret_cast<uint32_t*>(dst + 128) = w[1];
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (base + (j >> 2) * 128 + 4 * lane + (j & 3) < n1)
        dst[(j >> 2) * 128 + (j & 3)] = static_cast<uint8_t>(w[j >> 2] >> (8 * (j & 3)));
  }
}


// ---------------------------------------------------------------------------
// bf16 encoder.  CTA = 8 compute warps + 1 producer warp.  Whole chunks of
// 8192 elements (128 blocks) stream into a 3-stage ring by 1-D bulk copies;
// two threads own one 64-block (32 elements each).  A warp copies its 2 KB
// of a stage into registers and releases the stage at once (per-warp release
// barrier, no CTA-wide barrier in the loop).  Per pair of elements the fast
// path is: unpack, t = x/s, the bucket index and t - midpoint in packed f32x2
// arithmetic, two 8-byte bucket loads from this lane's copy of the table, and
// code = (codes below the bucket + 1) + (sign of t - midpoint).  The block's
// absmax is a packed 16-bit integer max of the bf16 magnitudes (bits of |w|;
// an exponent field of all ones means Inf or NaN).  Blocks whose scale would
// make 1/s leave the normal range, and blocks with an element within 2^-17 of
// its stored midpoint, take the exact path (encode32_exact).  Blocks past
// the last whole chunk are left to the generic per-lane code (encode16).
// ---------------------------------------------------------------------------
constexpr int kBfChunkBlocks = 128;
constexpr int kDqMidBytes = 2048;   // 254 fp64 midpoints, staged in the ring for the DQ stage
constexpr int kBfChunkElems = kBfChunkBlocks * kBlock;   // 8192
constexpr int kBfStages = 3;
constexpr int kBfComputeWarps = 8;
constexpr int kBfThreads = (kBfComputeWarps + 1) * 32;
constexpr size_t kBfSmem = static_cast<size_t>(kBfStages) * kBfChunkElems * 2 + 128;
static_assert(kDqMidBytes >= 254 * 8 && kDqMidBytes % 16 == 0 &&
                  kDqMidBytes + 2 * kT8SignCells <= kBfStages * kBfChunkElems * 2,
              "DQ stage tables fit the ring");

// Bucket entries for the packed path: per bucket and lane one 8-byte entry
// (fp32 midpoint or 4.0, then codes below the bucket + 1); lane l reads its
// own copy at byte 256 * bucket + 8 * l (load_buckets fills them).

__device__ __forceinline__ uint64_t f2pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}

// Exact codes of 32 bf16 elements (read again from global memory: this path
// is rare) for scale s: the careful bucket search with the fp64 check near
// every midpoint, with s and the elements moved into the normal range of 1/s
// when needed.
__device__ __noinline__ uint4 encode32_exact(const uint16_t* __restrict__ gsrc, float s,
                                             const uint2* tab8, const double* mexact) {
  float sc = 1.0f;
  if (s < 1.17549435e-38f) sc = 18446744073709551616.0f;
  if (s > 8.50705917e37f) sc = 5.42101086e-20f;
  const float s_eff = s * sc;
  float inv_s;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(inv_s) : "f"(s_eff));
  uint32_t out[4] = {0u, 0u, 0u, 0u};
  for (int e = 0; e < 32; ++e) {
    const float x = bf16_bits_to_f32(__ldg(gsrc + e)) * sc;
    const float t = x * inv_s;
    int b = __float2int_rd(fmaf(t, 16.0f, 16.5f));
    b = b < 0 ? 0 : (b > kBuckets - 1 ? kBuckets - 1 : b);
    const uint2 ent = tab8[32 * b];
    const int jlo = static_cast<int>(ent.y) - 1;
    const float d = t - __uint_as_float(ent.x);
    uint32_t code = static_cast<uint32_t>(jlo) + (d > 0.0f ? 1u : 0u);
    if (fabsf(d) < kNearEps) code = exact_code(x, s_eff, jlo, mexact);
    // element e: word e / 8, byte (e % 8) / 2, high nibble for even e
    out[e >> 3] |= code << (8 * ((e & 7) >> 1) + ((e & 1) ? 0 : 4));
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

template <bool kDQ>
__global__ void __launch_bounds__(kBfThreads) nf4_encode_bf16_kernel(
    const uint16_t* __restrict__ W, int64_t numel, int64_t n1, uint8_t* __restrict__ packed,
    float* __restrict__ scales, unsigned long long* __restrict__ bins,
    unsigned int* __restrict__ done_ctas, float* __restrict__ offset_out,
    uint8_t* __restrict__ code8, float* __restrict__ s2, int32_t* d_status,
    unsigned long long token) {
  extern __shared__ uint8_t esm_raw[];
  uint16_t* ring = reinterpret_cast<uint16_t*>((reinterpret_cast<uintptr_t>(esm_raw) + 127) &
                                               ~static_cast<uintptr_t>(127));
  __shared__ uint2 tab8[kBuckets * 32];
  __shared__ uint32_t tab4[kBuckets * 32];
  __shared__ double mexact[15];
  __shared__ unsigned long long sbins[kDQ ? 256 : 1];
  __shared__ uint64_t full_bar[kBfStages];
  __shared__ uint64_t empty_bar[kBfStages];
  __shared__ int abort_flag;
  __shared__ int last_cta;
  __shared__ int krange[2];
  __shared__ long long chunk_of[kBfStages];   // the chunk in each stage; -1: no more
  pdl_launch_dependents();
  load_buckets(tab4, tab8, mexact);
  if (kDQ)
    for (int i = threadIdx.x; i < 256; i += blockDim.x) sbins[i] = 0ull;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kBfStages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], kBfComputeWarps);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();   // the tables above read no global memory
  if (kDQ) ws_clear_and_publish(bins, done_ctas, token);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nchunks = numel / kBfChunkElems;
  constexpr uint32_t kChunkBytes = kBfChunkElems * 2;
  BinCache bc;
  bool bad = false;

  if (warp == kBfComputeWarps) {
    // ------------------------------ producer ------------------------------
    // Chunk j of this CTA: blockIdx.x + j * gridDim.x for the first
    // kBfStages (and all of them without a workspace); then, with a workspace
    // (kDQ), the next unclaimed chunk past those waves from the call's
    // counter, so that CTAs that stream faster take more chunks.  The chunk
    // goes to the compute warps with the stage; -1 (with a plain arrival)
    // ends their loop.
    if (lane == 0) {
      uint32_t last_parity[kBfStages];
      for (int s = 0; s < kBfStages; ++s) last_parity[s] = 2;
      bool counter_ready = false;
      for (int64_t j = 0;; ++j) {
        const int s = static_cast<int>(j % kBfStages);
        const uint32_t ph = static_cast<uint32_t>((j / kBfStages) & 1);
        if (j >= kBfStages && !mbar_wait(&empty_bar[s], ph ^ 1)) { abort_flag = 1; break; }
        int64_t c = blockIdx.x + j * static_cast<int64_t>(gridDim.x);
        if (kDQ && j >= kBfStages) {
          if (!counter_ready) {
            counter_ready = ws_wait_published(bins, token);   // CTA 0 cleared the counter
            if (!counter_ready) { abort_flag = 1; break; }
          }
          c = kBfStages * static_cast<int64_t>(gridDim.x) +
              static_cast<int64_t>(atomicAdd(ws_chunk_counter(bins), 1ull));
        }
        if (c >= nchunks) {
          chunk_of[s] = -1;
          mbar_arrive(&full_bar[s]);
          last_parity[s] = 2;   // the stage's last copy was consumed (the wait above)
          break;
        }
        chunk_of[s] = c;
        mbar_arrive_expect_tx(&full_bar[s], kChunkBytes);
        bulk_load_1d(ring + s * kBfChunkElems, W + c * kBfChunkElems, kChunkBytes, &full_bar[s]);
        last_parity[s] = ph;
      }
      // every copy issued has landed before the CTA can exit
      for (int s = 0; s < kBfStages; ++s)
        if (last_parity[s] < 2 && !mbar_wait(&full_bar[s], last_parity[s])) abort_flag = 1;
    }
  } else {
    // ---------------------------- compute warps ----------------------------
    const int half = lane & 1;
    const int lb = (threadIdx.x >> 1);                  // block within the chunk
    const uint32_t tb = smem_u32(tab8) + static_cast<uint32_t>(lane) * 8u - 0x4B000000u * 256u;
    const uint64_t c16 = f2pack(8388624.0f, 8388624.0f);   // 2^23 + 16 in each lane of the pair
    const uint64_t k16 = f2pack(16.0f, 16.0f);
    for (int64_t j = 0;; ++j) {
      const int s = static_cast<int>(j % kBfStages);
      const uint32_t ph = static_cast<uint32_t>((j / kBfStages) & 1);
      if (!mbar_wait(&full_bar[s], ph)) { abort_flag = 1; break; }
      const int64_t c = *reinterpret_cast<volatile long long*>(&chunk_of[s]);
      if (c < 0) break;
      const uint16_t* src = ring + s * kBfChunkElems + lb * kBlock + half * 32;
      // The thread's 64 bytes are four 16-byte chunks; slot v reads chunk
      // (v + rot) & 3, so that the 8 lanes of a quarter warp (4 blocks 128
      // bytes apart) read 8 different bank groups.  Codes are formed in slot
      // order and the packed words rotated back before the store.
      const int rot = (lane >> 1) & 3;
      uint32_t w[16];
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 q = *reinterpret_cast<const uint4*>(src + 8 * ((v + rot) & 3));
        w[4 * v] = q.x; w[4 * v + 1] = q.y; w[4 * v + 2] = q.z; w[4 * v + 3] = q.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[s]);
      const int64_t blk = c * kBfChunkBlocks + lb;
      // absmax: largest bf16 magnitude of the block (the pair of threads)
      uint32_t m2 = 0u;
#pragma unroll
      for (int i = 0; i < 16; ++i)
        asm("max.u16x2 %0, %0, %1;" : "+r"(m2) : "r"(w[i] & 0x7FFF7FFFu));
      uint32_t amb = max(m2 & 0xFFFFu, m2 >> 16);
      amb = max(amb, __shfl_xor_sync(0xFFFFFFFFu, amb, 1));
      const bool finite = amb < 0x7F80u;
      bad |= !finite;
      const float s_ = (finite && amb != 0u) ? __uint_as_float(amb << 16) : 1.0f;
      uint32_t out[4] = {0x77777777u, 0x77777777u, 0x77777777u, 0x77777777u};
      if (finite) {
        if (s_ < 1.17549435e-38f || s_ > 8.50705917e37f) {
          const uint4 ex = encode32_exact(W + blk * kBlock + half * 32, s_, tab8, mexact);
          out[0] = ex.x; out[1] = ex.y; out[2] = ex.z; out[3] = ex.w;
        } else {
          float inv_s;
          asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(inv_s) : "f"(s_));
          const uint64_t inv2 = f2pack(inv_s, inv_s);
          float dmin = 1.0f;
#pragma unroll
          for (int q = 0; q < 4; ++q) out[q] = 0u;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint64_t x2 = f2pack(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
            uint64_t t2, y2;
            asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(t2) : "l"(x2), "l"(inv2));
            asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(y2) : "l"(t2), "l"(k16), "l"(c16));
            float y0, y1;
            f2unpack(y2, y0, y1);
            uint32_t m0, j0, m1, j1;
            asm("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(m0), "=r"(j0) : "r"(tb + __float_as_uint(y0) * 256u));
            asm("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(m1), "=r"(j1) : "r"(tb + __float_as_uint(y1) * 256u));
            uint64_t d2;
            asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d2) : "l"(t2), "l"(f2pack(__uint_as_float(m0), __uint_as_float(m1))));
            float d0, d1;
            f2unpack(d2, d0, d1);
            dmin = fminf(dmin, fminf(fabsf(d0), fabsf(d1)));
            const uint32_t code0 = j0 + static_cast<uint32_t>(__float_as_int(d0) >> 31);
            const uint32_t code1 = j1 + static_cast<uint32_t>(__float_as_int(d1) >> 31);
            // elements 2i (high nibble) and 2i + 1 of byte i % 4 of word i / 4
            out[i >> 2] += ((code0 << 4) | code1) << (8 * (i & 3));
          }
          // word v belongs to chunk (v + rot) & 3: rotate back in two steps
          uint32_t o1[4];
#pragma unroll
          for (int v = 0; v < 4; ++v) o1[v] = (rot & 1) ? out[(v + 3) & 3] : out[v];
#pragma unroll
          for (int v = 0; v < 4; ++v) out[v] = (rot & 2) ? o1[(v + 2) & 3] : o1[v];
          if (dmin < kNearEps) {
            const uint4 ex = encode32_exact(W + blk * kBlock + half * 32, s_, tab8, mexact);
            out[0] = ex.x; out[1] = ex.y; out[2] = ex.z; out[3] = ex.w;
          }
        }
      }
      *reinterpret_cast<uint4*>(packed + blk * (kBlock / 2) + half * 16) =
          make_uint4(out[0], out[1], out[2], out[3]);
      if (half == 0) scales[blk] = s_;
      if (kDQ) {
        // exponent bins of the warp's 16 block scales, summed exactly by two
        // warp reductions.  Bin k counts units of 2^(k-150); a scale is a bf16
        // magnitude m8 * 2^(key-134) (m8 its 8-bit significand), which is
        // m8 << (16 + key - kb) units of bin kb.  With kb = the warp's largest
        // key - 3 (at least 1), every scale within 16 binades of kb is an
        // integer below 2^27 there, and the 16 of them sum below 2^31: one
        // shared atomic per warp and chunk.  Scales further below go to their
        // own bins, one atomic each.
        const uint32_t u = __float_as_uint(s_);
        const uint32_t E = (u >> 23) & 0xFFu;
        const uint32_t key = half == 0 ? (E ? E : 1u) : 0u;   // odd lanes carry no scale
        const uint32_t kmax = __reduce_max_sync(0xFFFFFFFFu, key);
        const uint32_t kb = kmax > 4u ? kmax - 3u : 1u;
        const uint32_t m8 = ((u >> 16) & 0x7Fu) | (E ? 0x80u : 0u);
        const bool near = key + 16u >= kb;
        const uint32_t sum = __reduce_add_sync(0xFFFFFFFFu, half == 0 && near ? m8 << (16u + key - kb) : 0u);
        if (lane == 0) atomicAdd(&sbins[kb], static_cast<unsigned long long>(sum));
        if (half == 0 && !near) atomicAdd(&sbins[key], static_cast<unsigned long long>(m8) << 16);
      }
    }
  }
  __syncthreads();
  if (abort_flag && threadIdx.x == 0) raise_status(d_status, QLORA_ERR_TIMEOUT);
  // blocks not covered by whole chunks: the generic path, 4 lanes per block
  {
    const int sub = lane & 3;
    const unsigned gmask = 0xFu << (lane & 28);
    const int64_t first = nchunks * kBfChunkBlocks;
    const int64_t ngroups = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 2;
    const bool aligned16 = (reinterpret_cast<uintptr_t>(W) & 15u) == 0;
    for (int64_t blk = first + ((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 2);
         blk < n1; blk += ngroups) {
      const int64_t e0 = blk * kBlock + sub * kLaneElems;
      const bool full = e0 + kLaneElems <= numel;
      float x[kLaneElems];
      load16<uint16_t>(W, e0, numel, full && aligned16, x);
      encode16<kDQ>(x, blk, e0, sub, gmask, numel, full, tab4, mexact, packed, scales, bc, sbins, bad);
    }
  }
  if (bad) raise_status(d_status, QLORA_ERR_NONFINITE);
  if (kDQ) {
    bc.flush(sbins);
    __shared__ int published;
    __syncthreads();
    if (threadIdx.x == 0) {
      published = ws_wait_published(bins, token) ? 1 : 0;
      if (!published) raise_status(d_status, QLORA_ERR_TIMEOUT);
    }
    __syncthreads();
    if (published)
      for (int i = threadIdx.x; i < 256; i += blockDim.x)
        if (sbins[i]) atomicAdd(&bins[i], sbins[i]);
    __syncthreads();
    if (offset_out == nullptr) return;   // a shard: the caller adds the bins of all shards
    if (threadIdx.x == 0) {
      __threadfence();
      last_cta = atomicAdd(done_ctas, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (last_cta) {
      __threadfence();
      for (int i = threadIdx.x; i < 256; i += blockDim.x) sbins[i] = __ldcg(bins + i);
      __syncthreads();
      bins_key_range(sbins, krange);
      __syncthreads();
      if (threadIdx.x == 0) {
        *offset_out = __uint_as_float(exact_mean_bits(sbins, krange[0], krange[1], n1));
        if (code8 != nullptr) {
          __threadfence();
          asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(ws_mean_flag(bins)), "l"(token)
                       : "memory");
        }
      }
    }
    if (code8 == nullptr) return;
    // Double quantization in the same launch.  Every CTA of the grid is
    // resident (one wave, sized by the occupancy of this kernel), so each
    // waits for the last CTA's mean (bounded) and then encodes groups of 256
    // scales, one warp per group.  The ring is free: every copy has landed
    // and been read.
    double* mid = reinterpret_cast<double*>(ring);
    uint8_t* cells = reinterpret_cast<uint8_t*>(ring) + kDqMidBytes;
    for (int k = threadIdx.x; k < 254; k += blockDim.x) mid[k] = kT8Mid.m[k];
    for (int k = threadIdx.x; k < 2 * kT8SignCells / 16; k += blockDim.x)
      reinterpret_cast<uint4*>(cells)[k] = reinterpret_cast<const uint4*>(kT8Cells.k0)[k];
    __shared__ float s_mean;
    if (threadIdx.x == 0) {
      published = ws_wait_mean(bins, token) ? 1 : 0;
      if (published)
        s_mean = __ldcg(offset_out);
      else
        raise_status(d_status, QLORA_ERR_TIMEOUT);
    }
    __syncthreads();
    if (!published) return;
    const int nwarps = kBfComputeWarps + 1;
    const int64_t n2 = (n1 + kDQBlock - 1) / kDQBlock;
    for (int64_t g = static_cast<int64_t>(blockIdx.x) * nwarps + warp; g < n2;
         g += static_cast<int64_t>(gridDim.x) * nwarps)
      dq_encode_group(scales, n1, g, s_mean, mid, cells, code8, s2, lane);
  }
}

// One warp per group of 256 scales, 8 groups per CTA (fp32 weights, and the
// shards of a sharded quantization, whose mean is formed after all shards).
__global__ void __launch_bounds__(256) dq_encode_kernel(const float* __restrict__ a, int64_t n1,
                                                        const float* __restrict__ offset_p,
                                                        uint8_t* __restrict__ code8,
                                                        float* __restrict__ s2) {
  __shared__ float s_off;
  __shared__ double mid[254];
  __shared__ __align__(16) uint8_t cells[2 * kT8SignCells];
  pdl_launch_dependents();
  for (int k = threadIdx.x; k < 254; k += blockDim.x) mid[k] = kT8Mid.m[k];
  for (int k = threadIdx.x; k < 2 * kT8SignCells / 16; k += blockDim.x)
    reinterpret_cast<uint4*>(cells)[k] = reinterpret_cast<const uint4*>(kT8Cells.k0)[k];
  __syncthreads();
  pdl_wait();   // the tables above read only compile-time constants
  if (threadIdx.x == 0) s_off = *offset_p;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t n2 = (n1 + kDQBlock - 1) / kDQBlock;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * 8 + warp; g < n2;
       g += static_cast<int64_t>(gridDim.x) * 8)
    dq_encode_group(a, n1, g, s_off, mid, cells, code8, s2, lane);
}

// The exact mean of n1 first-level scales from exponent bins that already
// hold every shard's sums (sharded quantization): one CTA.
__global__ void __launch_bounds__(256) dq_mean_kernel(const unsigned long long* __restrict__ bins,
                                                      int64_t n1, float* __restrict__ offset_out) {
  __shared__ unsigned long long sb[256];
  __shared__ int krange[2];
  pdl_launch_dependents();
  pdl_wait();
  sb[threadIdx.x] = bins[threadIdx.x];
  __syncthreads();
  bins_key_range(sb, krange);
  __syncthreads();
  if (threadIdx.x == 0) *offset_out = __uint_as_float(exact_mean_bits(sb, krange[0], krange[1], n1));
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
// ---------------------------------------------------------------------------
// Uniform signed INT4 (the comparator codebook; page "SFT（四）：QLoRA的4-bit量化与
// LoRA微调原理", §6 先理解最普通的分块量化): per 64-block s = amax / 7 (formed in
// fp64, stored as fp32; 1 for an all-zero block), q = clip(round(w / s), -7, 7)
// with w / s in fp64 and ties away from zero, code q + 8; an odd tail is padded
// with code 8.  One thread per block: 64 fp64 divisions, a comparator path.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) int4_encode_kernel(const T* __restrict__ W, int64_t numel,
                                                          uint8_t* __restrict__ packed,
                                                          float* __restrict__ scales,
                                                          int32_t* d_status) {
  pdl_launch_dependents();
  pdl_wait();
  const int64_t n1 = (numel + kBlock - 1) / kBlock;
  const int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (b >= n1) return;
  const int64_t e0 = b * kBlock;
  const int cnt = static_cast<int>(numel - e0 < kBlock ? numel - e0 : kBlock);
  float x[kBlock];
#pragma unroll
  for (int i = 0; i < kBlock; ++i) {
    float v = 0.0f;
    if (i < cnt) {
      if constexpr (sizeof(T) == 2) v = bf16_bits_to_f32(W[e0 + i]);
      else v = W[e0 + i];
    }
    x[i] = v;
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < kBlock; ++i) amax = fmax_nan(amax, fabsf(x[i]));
  if (!(amax <= FLT_MAX)) {
    raise_status(d_status, QLORA_ERR_NONFINITE);
    amax = 0.0f;
  }
  const float sc = amax > 0.0f ? __double2float_rn(__ddiv_rn(static_cast<double>(amax), 7.0)) : 1.0f;
  scales[b] = sc;
  const double sd = static_cast<double>(sc);
  uint32_t words[kBlock / 8];
#pragma unroll
  for (int wi = 0; wi < kBlock / 8; ++wi) {
    uint32_t w = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int i = wi * 8 + k;
      uint32_t code = static_cast<uint32_t>(kPadCodeInt4);
      if (i < cnt) {
        const double t = __ddiv_rn(static_cast<double>(x[i]), sd);
        const double r = floor(__dadd_rn(fabs(t), 0.5));
        const int q = static_cast<int>(fmin(r, 7.0)) * (t >= 0.0 ? 1 : -1);
        code = static_cast<uint32_t>(q + 8);
      }
      // byte k/2 of the word: element 2m in the high nibble, 2m+1 in the low
      w |= code << (8 * (k >> 1) + ((k & 1) ? 0 : 4));
    }
    words[wi] = w;
  }
  const int64_t nbytes = (numel + 1) >> 1;
  const int64_t b0 = e0 >> 1;
  if (cnt == kBlock) {
    uint4* dst = reinterpret_cast<uint4*>(packed + b0);
    dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
    dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
  } else {
    for (int k = 0; k < kBlock / 2; ++k)
      if (b0 + k < nbytes) packed[b0 + k] = static_cast<uint8_t>(words[k >> 2] >> (8 * (k & 3)));
  }
}

namespace {

// The NF4 encoder over `numel` elements of W: packed bytes, one fp32 scale per
// 64-block into `scales`, and (dq) the scales' exponent bins; with
// `offset_out` the last CTA also forms their exact mean there.
cudaError_t launch_encoder(const void* W, int dtype, int64_t numel, uint8_t* packed, float* scales,
                           bool dq, unsigned long long* bins, unsigned int* done_ctas,
                           float* offset_out, uint8_t* code8, float* s2, int32_t* d_status,
                           cudaStream_t st, int num_sms) {
  // a token per call (never repeated within the process): the kernel's CTA 0
  // publishes it once it has cleared the workspace head
  static std::atomic<unsigned long long> next_token{0x9E3779B97F4A7C15ull};
  const unsigned long long token = next_token.fetch_add(1ull);
  const int64_t n1 = (numel + kBlock - 1) / kBlock;
  const int threads = 256;
  const int64_t want = (n1 * 4 + threads - 1) / threads;
  ProfScope prof(kProfQuantize, st);
  // one wave of resident CTAs (each loops over chunks); attributes and
  // occupancy per device
  static int per_sm[kMaxDevices][4];
  static DeviceOnce once;
  cudaError_t e = once.run([&](int dev) {
    const int b16 = static_cast<int>(encode_smem_bytes<uint16_t>());
    const int b32 = static_cast<int>(encode_smem_bytes<float>());
    (void)b16;
    const void* fns[4] = {reinterpret_cast<const void*>(nf4_encode_bf16_kernel<false>),
                          reinterpret_cast<const void*>(nf4_encode_bf16_kernel<true>),
                          reinterpret_cast<const void*>(nf4_encode_kernel<float, false>),
                          reinterpret_cast<const void*>(nf4_encode_kernel<float, true>)};
    for (int i = 0; i < 4; ++i) {
      const int bytes = i < 2 ? static_cast<int>(kBfSmem) : b32;
      const int nthr = i < 2 ? kBfThreads : threads;
      cudaError_t r = cudaFuncSetAttribute(fns[i], cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
      if (r != cudaSuccess) return r;
      cudaFuncSetAttribute(fns[i], cudaFuncAttributePreferredSharedMemoryCarveout, 100);
      int nb = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fns[i], nthr, bytes) != cudaSuccess || nb < 1)
        nb = 1;
      per_sm[dev][i] = nb;
    }
    (void)cudaGetLastError();   // a refused carveout hint is not an error
    return cudaSuccess;
  });
  if (e != cudaSuccess) return e;
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  const int kind = (dtype == QLORA_DTYPE_BF16 ? 0 : 2) + (dq ? 1 : 0);
  const int64_t cap = static_cast<int64_t>(num_sms) * per_sm[dev][kind];
  const int blocks = static_cast<int>(want < cap ? want : cap);
  if (dtype == QLORA_DTYPE_BF16) {
    // whole 8192-element chunks per CTA iteration; at least one CTA per SM
    // for the ragged remainder
    const uint16_t* w16 = static_cast<const uint16_t*>(W);
    const int64_t chunks = numel / kBfChunkElems;
    const int64_t cap16 = static_cast<int64_t>(num_sms) * per_sm[dev][kind];
    int64_t g16 = chunks < cap16 ? chunks : cap16;
    const int64_t rem_groups = (n1 - chunks * kBfChunkBlocks + kBfThreads / 4 - 1) / (kBfThreads / 4);
    if (g16 < rem_groups) g16 = rem_groups < cap16 ? rem_groups : cap16;
    if (g16 < 1) g16 = 1;
    e = dq ? launch_pdl(nf4_encode_bf16_kernel<true>, dim3(static_cast<unsigned>(g16)), dim3(kBfThreads),
                        kBfSmem, st, 1, w16, numel, n1, packed, scales, bins, done_ctas, offset_out,
                        code8, s2, d_status, token)
           : launch_pdl(nf4_encode_bf16_kernel<false>, dim3(static_cast<unsigned>(g16)), dim3(kBfThreads),
                        kBfSmem, st, 1, w16, numel, n1, packed, scales, bins, done_ctas, offset_out,
                        code8, s2, d_status, token);
  } else {
    const size_t sm = encode_smem_bytes<float>();
    const float* w32 = static_cast<const float*>(W);
    e = dq ? launch_pdl(nf4_encode_kernel<float, true>, dim3(blocks), dim3(threads), sm, st, 1, w32,
                        numel, n1, packed, scales, bins, done_ctas, offset_out, d_status, token)
           : launch_pdl(nf4_encode_kernel<float, false>, dim3(blocks), dim3(threads), sm, st, 1, w32,
                        numel, n1, packed, scales, bins, done_ctas, offset_out, d_status, token);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  return e;
}

// Scale codes and second-level scales of n1 centred scales (groups of 256
// from the first), given the offset in device memory.
cudaError_t launch_dq_encode(const float* scales, int64_t n1, const float* offset, uint8_t* code8,
                             float* s2, cudaStream_t st, int num_sms) {
  const int64_t n2 = (n1 + kDQBlock - 1) / kDQBlock;
  ProfScope prof(kProfQuantize, st);
  const int64_t want_g = (n2 + 7) / 8;
  const int64_t grid = want_g < num_sms * 8LL ? want_g : num_sms * 8LL;
  cudaError_t e = launch_pdl(dq_encode_kernel, dim3(static_cast<unsigned>(grid)), dim3(256), 0, st,
                             1, scales, n1, offset, code8, s2);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_int4(const void* W, int dtype, int64_t numel, uint8_t* packed, float* scales,
                        int32_t* d_status, cudaStream_t st) {
  const int64_t n1 = (numel + kBlock - 1) / kBlock;
  const dim3 grid(static_cast<unsigned>((n1 + 255) / 256));
  ProfScope prof(kProfQuantize, st);
  const cudaError_t e1 =
      dtype == QLORA_DTYPE_BF16
          ? launch_pdl(int4_encode_kernel<uint16_t>, grid, dim3(256), 0, st, 1,
                       static_cast<const uint16_t*>(W), numel, packed, scales, d_status)
          : launch_pdl(int4_encode_kernel<float>, grid, dim3(256), 0, st, 1,
                       static_cast<const float*>(W), numel, packed, scales, d_status);
  if (e1 != cudaSuccess) return e1;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(const void* W, int dtype, int64_t numel, uint8_t* packed,
                            float* absmax_out, bool dq, uint8_t* code8, float* s2, float* offset,
                            void* ws, int32_t* d_status, cudaStream_t st, int num_sms,
                            int codebook) {
  // uniform INT4: no double quantization, no workspace
  if (codebook == 1) return launch_int4(W, dtype, numel, packed, absmax_out, d_status, st);
  if (!dq)
    return launch_encoder(W, dtype, numel, packed, absmax_out, false, nullptr, nullptr, nullptr,
                          nullptr, nullptr, d_status, st, num_sms);
  // workspace: 256 exponent bins, the finished-CTA counter, the call token and
  // the mean's flag, then the scales
  const int64_t n1 = (numel + kBlock - 1) / kBlock;
  unsigned long long* bins = static_cast<unsigned long long*>(ws);
  unsigned int* done_ctas = reinterpret_cast<unsigned int*>(static_cast<char*>(ws) + 2048);
  float* scales = reinterpret_cast<float*>(static_cast<char*>(ws) + kQuantizeWsHead);
  // bf16 weights: scale codes and second-level scales in the encoder's own
  // launch; fp32 weights: a second launch
  const bool fused = dtype == QLORA_DTYPE_BF16;
  cudaError_t e = launch_encoder(W, dtype, numel, packed, scales, true, bins, done_ctas, offset,
                                 fused ? code8 : nullptr, fused ? s2 : nullptr, d_status, st, num_sms);
  if (e != cudaSuccess || fused) return e;
  return launch_dq_encode(scales, n1, offset, code8, s2, st, num_sms);
}

cudaError_t launch_quantize_shard_begin(const void* W_shard, int dtype, int64_t numel_total,
                                        int64_t b0, int64_t b1, uint8_t* packed, float* absmax_out,
                                        bool dq, void* ws, int32_t* d_status, cudaStream_t st,
                                        int num_sms, int codebook) {
  const int64_t e_end = b1 * kBlock < numel_total ? b1 * kBlock : numel_total;
  const int64_t numel = e_end - b0 * kBlock;
  uint8_t* pk = packed + b0 * (kBlock / 2);
  if (codebook == 1) return launch_int4(W_shard, dtype, numel, pk, absmax_out + b0, d_status, st);
  if (!dq)
    return launch_encoder(W_shard, dtype, numel, pk, absmax_out + b0, false, nullptr, nullptr,
                          nullptr, nullptr, nullptr, d_status, st, num_sms);
  unsigned long long* bins = static_cast<unsigned long long*>(ws);
  float* scales = reinterpret_cast<float*>(static_cast<char*>(ws) + kQuantizeWsHead);
  return launch_encoder(W_shard, dtype, numel, pk, scales, true, bins, nullptr, nullptr, nullptr,
                        nullptr, d_status, st, num_sms);
}

cudaError_t launch_quantize_shard_end(int64_t numel_total, int64_t b0, int64_t b1, const void* ws,
                                      uint8_t* code8, float* s2, float* offset, cudaStream_t st,
                                      int num_sms) {
  const int64_t n1 = (numel_total + kBlock - 1) / kBlock;
  const unsigned long long* bins = static_cast<const unsigned long long*>(ws);
  const float* scales =
      reinterpret_cast<const float*>(static_cast<const char*>(ws) + kQuantizeWsHead);
  cudaError_t e;
  {
    ProfScope prof(kProfQuantize, st);
    e = launch_pdl(dq_mean_kernel, dim3(1), dim3(256), 0, st, 1, bins, n1, offset);
    if (e == cudaSuccess) e = cudaGetLastError();
  }
  if (e != cudaSuccess || b1 <= b0) return e;
  return launch_dq_encode(scales, b1 - b0, offset, code8 + b0, s2 + b0 / kDQBlock, st, num_sms);
}

size_t quantize_workspace_bytes(int64_t numel, bool dq) {
  if (!dq) return 0;
  const int64_t n1 = (numel + kBlock - 1) / kBlock;
  return kQuantizeWsHead + static_cast<size_t>(n1) * 4;
}

}  // namespace qnf4
