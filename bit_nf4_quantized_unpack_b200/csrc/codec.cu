// codec.cu -- NF4 quantization with double-quantized constants, and the standalone
// double dequantization (page "QLoRA", itwiki.kr, sections "4비트 NormalFloat(NF4)" and
// "이중 양자화"). All three kernels are HBM-bound streaming passes.
#include <cuda_bf16.h>

#include <atomic>

#include "internal.h"
#include "nf4_device.cuh"

namespace qlora {
namespace {

static_assert(kT8Entries == kT8Size, "one T8 table size for the host and the device");
constexpr int kQuantThreads = 256;
constexpr int kMaxQuantCtas = 148 * 8;

// Eight consecutive weights as loaded (kept raw until they are used, so that a prefetch
// does not wait for its data) and their fp32 values.
template <typename T>
struct Raw8;
template <>
struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = __ldg(reinterpret_cast<const float4*>(p));
    b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ __forceinline__ void values(float (&v)[8]) const {
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
};
template <>
struct Raw8<uint16_t> {  // bf16
  uint4 a;
  __device__ __forceinline__ void load(const uint16_t* p) { a = __ldg(reinterpret_cast<const uint4*>(p)); }
  __device__ __forceinline__ void values(float (&v)[8]) const {
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};

// NF4 code of x in [-1, 1] from the bucket table in shared memory, given
// bk = fl32(16 x + 16 + 1.5 * 2^23): that number lies in [2^23, 2^24), where the ulp is 1,
// so its low mantissa bits hold the bucket round-half-even(16 x + 16) (0..32). The table
// is two arrays of 64 4-byte words (negated fp32 thresholds, codes) at a fixed distance,
// so that one address serves both loads, indexed by the low six bits of bk: any bit
// pattern (a NaN from a non-finite input) stays inside it. Entries 33-63 are -inf
// (no threshold) and code 0.
constexpr int kBucketSlots = 64;
struct BucketSmem {
  float nthr[kBucketSlots];  // -threshold
  uint32_t code[kBucketSlots];
};
constexpr float kBucketBias = 16.0f + 12582912.0f;  // S + 1.5 * 2^23
__device__ __forceinline__ uint32_t bucket_index(float bk) {
  return __float_as_uint(bk) & (kBucketSlots - 1);
}
__device__ __forceinline__ uint32_t bucket_code(float x, const BucketSmem& sb) {
  const uint32_t idx = bucket_index(__fmaf_rn(x, static_cast<float>(kBucketScale), kBucketBias));
  return sb.code[idx] + (-x <= sb.nthr[idx] ? 1u : 0u);
}

// Eight codes packed as one 32-bit word (element 2j in the low nibble of byte j, 2j+1 in
// the high one) from the bucket codes cw[i] (0..15, low byte) and d[i] = fl32(x_i -
// thr_i): x >= thr exactly when d is not negative (the sign of a rounded difference is
// that of the exact one, and x == thr gives +0; no threshold is zero), and then the code
// is one above the bucket's (at most 14 where the bucket holds a threshold, so the
// nibble does not carry). The sign bytes come from prmt's sign-replicating selectors
// (0xFF where d < 0).
__device__ __forceinline__ uint32_t pack_codes8(const uint32_t (&cw)[8], const float (&d)[8]) {
  const uint32_t ce = prmt(prmt(cw[0], cw[2], 0x0040u), prmt(cw[4], cw[6], 0x0040u), 0x5410u);
  const uint32_t co = prmt(prmt(cw[1], cw[3], 0x0040u), prmt(cw[5], cw[7], 0x0040u), 0x5410u);
  uint32_t di[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) di[i] = __float_as_uint(d[i]);
  const uint32_t se = prmt(prmt(di[0], di[2], 0x00FBu), prmt(di[4], di[6], 0x00FBu), 0x5410u);
  const uint32_t so = prmt(prmt(di[1], di[3], 0x00FBu), prmt(di[5], di[7], 0x00FBu), 0x5410u);
  const uint32_t neg = (se & 0x0F0F0F0Fu) | (so & 0xF0F0F0F0u);  // 0xF where x < thr
  return ce + (co << 4) + (0x11111111u & ~neg);
}

// max(|a|, |b|, |c|) in one three-input max (sm_100).
__device__ __forceinline__ float absmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(fabsf(a)), "f"(fabsf(b)), "f"(fabsf(c)));
  return d;
}

// fl32(S / n), rounded once to nearest (ties to even), for S >= 0 exact in fp64 and
// 1 <= n < 2^53. q = fl64(S / n) is within half an fp64 ulp of S / n, so the correctly
// rounded fp32 is fl32(q) or a neighbour: only where S / n lies on the other side of
// (or on) an fp32 midpoint m around q can they differ, and the sign of m n - S, exact
// from one fused multiply-add (m has at most 25 significant bits), tells which.
__device__ float round_div_f32(double S, int64_t n) {
  const double dn = static_cast<double>(n);
  const double q = S / dn;
  float f = __double2float_rn(q);
  const float up = __uint_as_float(__float_as_uint(f) + 1u);
  const double m_hi = 0.5 * (static_cast<double>(f) + static_cast<double>(up));
  const double d_hi = fma(m_hi, dn, -S);  // < 0: S / n above the midpoint
  if (d_hi < 0.0 || (d_hi == 0.0 && (__float_as_uint(f) & 1u))) return up;
  if (f > 0.f) {
    const float dnv = __uint_as_float(__float_as_uint(f) - 1u);
    const double m_lo = 0.5 * (static_cast<double>(dnv) + static_cast<double>(f));
    const double d_lo = fma(m_lo, dn, -S);  // > 0: S / n below the midpoint
    if (d_lo > 0.0 || (d_lo == 0.0 && (__float_as_uint(f) & 1u))) return dnv;
  }
  return f;
}

// fl32(S / n) (round to nearest, ties to even) for S = sum_e bins[e] * 2^(e - 150), the
// exact sum of the block constants, and n >= 1 of them (n < 2^32). Exact integer
// arithmetic on 32-bit digits: A = S * 2^150 (< 2^311) scaled by 2^64 fills 14 digits;
// the quotient q = floor(A * 2^64 / n) then holds S / n as q * 2^-214 to at least 33
// significant bits, and the bits of q below the kept 24 (or below 2^-149 for a
// subnormal result) with the remainder decide the rounding.
// The CTA's threads add the bins into per-digit 64-bit sums (`acc`, 16 entries, zeroed
// by the caller; bin e adds to three digits, and no digit sum can reach 2^41), then
// thread 0 propagates the carries and divides; returns the mean in thread 0.
__device__ float exact_mean_f32(const unsigned long long* bins, int64_t n,
                                unsigned long long* acc) {
  constexpr int kD = 14;
  for (int e = 1 + threadIdx.x; e < 256; e += blockDim.x) {
    const unsigned long long v = bins[e];
    if (!v) continue;
    const int w = (e + 64) >> 5, sh = (e + 64) & 31;  // v * 2^(e + 64)
    atomicAdd(acc + w, (v << sh) & 0xFFFFFFFFull);
    atomicAdd(acc + w + 1, (v >> (32 - sh)) & 0xFFFFFFFFull);
    if (sh) atomicAdd(acc + w + 2, v >> (64 - sh));
  }
  __syncthreads();
  if (threadIdx.x != 0) return 0.f;
  uint32_t d[kD];
  unsigned long long carry = 0;
#pragma unroll
  for (int k = 0; k < kD; ++k) {
    const unsigned long long t = acc[k] + carry;
    d[k] = static_cast<uint32_t>(t);
    carry = t >> 32;
  }
  // q = d / n from the most significant digit; each 64-by-32-bit step estimates the
  // quotient digit in fp64 (within one of the truth, as cur < n * 2^32 < 2^64) and
  // corrects it exactly
  const uint64_t nn = static_cast<uint64_t>(n);
  const double rn = 1.0 / static_cast<double>(nn);
  uint64_t rem = 0;
#pragma unroll
  for (int k = kD - 1; k >= 0; --k) {
    const uint64_t cur = (rem << 32) | d[k];
    uint64_t q = static_cast<uint64_t>(static_cast<double>(cur) * rn);
    if (q > 0xFFFFFFFFull) q = 0xFFFFFFFFull;
    int64_t r = static_cast<int64_t>(cur - q * nn);
    while (r < 0) {
      --q;
      r += static_cast<int64_t>(nn);
    }
    while (r >= static_cast<int64_t>(nn)) {
      ++q;
      r -= static_cast<int64_t>(nn);
    }
    d[k] = static_cast<uint32_t>(q);
    rem = static_cast<uint64_t>(r);
  }
  int top = -1;  // most significant set bit of q
#pragma unroll
  for (int k = kD - 1; k >= 0; --k)
    if (top < 0 && d[k]) top = 32 * k + 31 - __clz(d[k]);
  if (top < 0) return 0.f;
  auto dig = [&](int i) -> uint64_t {
    uint64_t v = 0;
#pragma unroll
    for (int k = 0; k < kD; ++k)
      if (k == i) v = d[k];
    return v;
  };
  auto nonzero_below = [&](int nbits) -> bool {  // any of q's bits 0 .. nbits - 1
    bool any = false;
#pragma unroll
    for (int k = 0; k < kD; ++k) {
      const int nb = min(32, nbits - 32 * k);
      if (nb > 0) any |= (d[k] & (nb >= 32 ? 0xFFFFFFFFu : ((1u << nb) - 1u))) != 0u;
    }
    return any;
  };
  if (top < 65) {  // below 2^-149: 0, or the smallest subnormal when above half of it
    const bool above_half = top == 64 && (rem != 0 || nonzero_below(64));
    return above_half ? __uint_as_float(1u) : 0.f;
  }
  // the 64-bit window of q whose top bit is bit `top` (bits top - 63 .. top)
  const int lo = top - 63;
  const int k0 = lo >> 5, sh = lo & 31;
  const uint64_t x = dig(k0) | (dig(k0 + 1) << 32), y = dig(k0 + 2);
  const uint64_t win = sh ? ((x >> sh) | (y << (64 - sh))) : x;
  // fp32 keeps bits [lsb, top]: 24 bits, or down to 2^-149 (bit 65 of q)
  const int lsb = max(top - 23, 65);
  const int nkeep = top - lsb + 1;  // 1 .. 24
  uint32_t sig = static_cast<uint32_t>(win >> (64 - nkeep));
  const uint32_t guard = static_cast<uint32_t>(win >> (63 - nkeep)) & 1u;
  const uint32_t sticky = (rem != 0 || nonzero_below(lsb - 1)) ? 1u : 0u;
  if (guard && (sticky || (sig & 1u))) ++sig;
  if (lsb == 65) return __uint_as_float(sig);  // subnormal (sig == 2^23: smallest normal)
  int ebits = top - 214 + 127;                   // biased exponent of the binade
  if (sig == 0x1000000u) {                       // rounding carried into the next binade
    sig >>= 1;
    ++ebits;
  }
  return __uint_as_float((static_cast<uint32_t>(ebits) << 23) | (sig & 0x7FFFFFu));
}

// Clears the accumulators of the mean (sum, exponent range, CTA counter) of level 1, its
// programmatic dependent, which waits for this grid before it reads its inputs. It is
// itself a programmatic dependent of the kernel before it on the stream and waits for it
// to complete before it writes.
__global__ void __launch_bounds__(32) k_quantize_prep(unsigned long long* acc) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (threadIdx.x < 4) acc[threadIdx.x] = 0ull;
}

// Level 1: one 64-block per group of kQuantLanes = 4 lanes (16 elements per lane). Writes
// the packed codes and the fp32 absmax of each block; the last CTA to finish forms the
// mean of all absmax, exactly: the CTAs add their absmax in fp64 and keep the smallest and
// largest exponent e (biased, 1 for subnormals) of the nonzero ones. Every absmax is then
// a multiple of g = 2^(e_min - 150) below 2^(e_max - 126), so when e_max - e_min +
// log2(n) <= 28 every partial sum is an integer multiple of g below 2^53 g: exact in
// fp64, whatever the order. The last CTA then rounds S / n to fp32 exactly
// (round_div_f32). Otherwise it re-reads all absmax and sums them as integers per
// exponent (exact_mean_f32). The sums and the counter are cleared by k_quantize_prep.
//
// x = fl32(w / absmax) is computed with Markstein's correction step (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000 processor", IBM J.
// Res. Dev. 34, 1990): with r = RN(1/m), q = RN(w r) and e = w - m q (exact in an FMA),
// RN(q + e r) is the correctly rounded quotient. Two weights go through each step at
// once in the packed f32x2 form. For m >= 2^-64, 1/m is finite and the
// residual stays exact for every |x| above 2^-36, far below the smallest threshold
// magnitude (0.04); blocks with a smaller absmax take plain IEEE division.
// The code of x comes from the bucket table: two shared-memory loads per weight, the
// threshold test as the sign of one f32x2 difference per two weights, and the byte
// permutes of pack_codes8 per eight.
constexpr int kQuantLanes = 4;
constexpr int kQuantPer = 64 / kQuantLanes;  // elements per lane
constexpr int kQuantChunks = kQuantPer / 8;  // 8-element loads (and 32-bit code words) per lane
template <typename T>
__global__ void __launch_bounds__(kQuantThreads)
    k_quantize_blocks(const T* __restrict__ W, int64_t nblocks,
                      const __grid_constant__ Nf4BucketTable tab, uint8_t* __restrict__ codes,
                      float* __restrict__ absmax, unsigned long long* __restrict__ acc_g,
                      float* __restrict__ mean_out) {
  const int lane = threadIdx.x & 31;
  const int sub = lane & (kQuantLanes - 1);
  const unsigned gmask = ((1u << kQuantLanes) - 1u) << (lane & (32 - kQuantLanes));
  const int64_t per_cta = kQuantThreads / kQuantLanes;
  __shared__ BucketSmem sb;
  __shared__ unsigned long long sbins[256];  // the wide-range mean of the last CTA
  for (int i = threadIdx.x; i < kBucketSlots; i += blockDim.x) {
    sb.nthr[i] = i < kCodeBuckets ? -tab.thr[i] : __int_as_float(0xFF800000);
    sb.code[i] = i < kCodeBuckets ? tab.code[i] : 0u;
  }
  __syncthreads();
  // the double quantization may be scheduled now; it waits for this grid's results
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // k_quantize_prep, and every kernel before it on the stream, is complete from here on:
  // W is ready, the accumulators are cleared, and no earlier call still reads the absmax
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t stride = static_cast<int64_t>(gridDim.x) * per_cta;
  int64_t b = blockIdx.x * per_cta + threadIdx.x / kQuantLanes;
  // this thread's part of the mean: fp64 sum and exponent range of its nonzero absmax
  double sum_d = 0.0;
  uint32_t e_lo = 255u, e_hi = 0u;
  // the next block's elements are in flight while this one is coded (one buffer: a second
  // one, rotated by register copies, measured slower)
  Raw8<T> n0[kQuantChunks];
#pragma unroll
  for (int h = 0; h < kQuantChunks; ++h)
    if (b < nblocks) n0[h].load(W + b * 64 + sub * kQuantPer + h * 8);
  for (; b < nblocks; b += stride) {
    float v[kQuantPer];
#pragma unroll
    for (int h = 0; h < kQuantChunks; ++h) n0[h].values(*reinterpret_cast<float(*)[8]>(v + 8 * h));
#pragma unroll
    for (int h = 0; h < kQuantChunks; ++h) {
      if (b + stride < nblocks) n0[h].load(W + (b + stride) * 64 + sub * kQuantPer + h * 8);
    }
    float m = fmaxf(fabsf(v[kQuantPer - 2]), fabsf(v[kQuantPer - 1]));
#pragma unroll
    for (int i = 0; i < kQuantPer - 2; i += 2) m = absmax3(m, v[i], v[i + 1]);
#pragma unroll
    for (int o = 1; o < kQuantLanes; o <<= 1) m = fmaxf(m, __shfl_xor_sync(gmask, m, o));
    uint32_t packed[kQuantChunks];
#pragma unroll
    for (int h = 0; h < kQuantChunks; ++h) packed[h] = 0u;
    if (m >= 0x1p-64f) {
      // the steps below on pairs of weights (packed f32x2: per lane the same roundings)
      const float r = __frcp_rn(m);
      const uint64_t rr = f2_pack(r, r), nm = f2_pack(-m, -m);
      const uint64_t kscale = f2_pack(kBucketScale, kBucketScale);
      const uint64_t kbias = f2_pack(kBucketBias, kBucketBias);
#pragma unroll
      for (int h = 0; h < kQuantChunks; ++h) {
        uint32_t cw[8];
        float d[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint64_t w = f2_pack(v[8 * h + 2 * i], v[8 * h + 2 * i + 1]);
          const uint64_t q = f2_mul(w, rr);
          const uint64_t e = f2_fma(q, nm, w);  // w - q m, exact
          const uint64_t x = f2_fma(e, rr, q);  // fl32(w / m)
          const uint64_t bk = f2_fma(x, kscale, kbias);
          float b0, b1;
          f2_unpack(bk, b0, b1);
          const uint32_t i0 = bucket_index(b0), i1 = bucket_index(b1);
          cw[2 * i] = sb.code[i0];
          cw[2 * i + 1] = sb.code[i1];
          const uint64_t df = f2_add(x, f2_pack(sb.nthr[i0], sb.nthr[i1]));  // fl32(x - thr)
          f2_unpack(df, d[2 * i], d[2 * i + 1]);
        }
        packed[h] = pack_codes8(cw, d);
      }
    } else {  // absmax zero or below 2^-64: plain IEEE division (x = 0 for a zero block)
#pragma unroll
      for (int i = 0; i < kQuantPer; ++i)
        packed[i / 8] |= bucket_code(m > 0.f ? __fdiv_rn(v[i], m) : 0.f, sb) << (4 * (i % 8));
    }
    if (kQuantChunks == 4)
      reinterpret_cast<uint4*>(codes + b * 32)[sub] =
          make_uint4(packed[0], packed[1 % kQuantChunks], packed[2 % kQuantChunks], packed[3 % kQuantChunks]);
    else
      reinterpret_cast<uint2*>(codes + b * 32)[sub] = make_uint2(packed[0], packed[1 % kQuantChunks]);
    if (sub == 0) {
      absmax[b] = m;
      const uint32_t e = __float_as_uint(m) >> 23;  // m >= 0
      const uint32_t eb = e ? e : 1u;
      sum_d += static_cast<double>(m);
      e_lo = m > 0.f ? min(e_lo, eb) : e_lo;
      e_hi = m > 0.f ? max(e_hi, eb) : e_hi;
    }
  }
  // the CTA's sum and range, then into the global accumulators
  __shared__ double red_d[kQuantThreads / 32];
  __shared__ uint32_t red_lo[kQuantThreads / 32], red_hi[kQuantThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sum_d += __shfl_xor_sync(0xFFFFFFFFu, sum_d, o);
    e_lo = min(e_lo, __shfl_xor_sync(0xFFFFFFFFu, e_lo, o));
    e_hi = max(e_hi, __shfl_xor_sync(0xFFFFFFFFu, e_hi, o));
  }
  if (lane == 0) {
    red_d[threadIdx.x / 32] = sum_d;
    red_lo[threadIdx.x / 32] = e_lo;
    red_hi[threadIdx.x / 32] = e_hi;
  }
  __syncthreads();
  __shared__ int last;
  if (threadIdx.x == 0) {
    double cs = 0.0;
    uint32_t lo = 255u, hi = 0u;
    for (int i = 0; i < kQuantThreads / 32; ++i) {
      cs += red_d[i];
      lo = min(lo, red_lo[i]);
      hi = max(hi, red_hi[i]);
    }
    atomicAdd(reinterpret_cast<double*>(acc_g), cs);
    atomicMax(reinterpret_cast<unsigned int*>(acc_g + 1), 255u - lo);  // cleared to 0
    atomicMax(reinterpret_cast<unsigned int*>(acc_g + 2), hi);
    __threadfence();
    last = atomicAdd(reinterpret_cast<unsigned int*>(acc_g + 3), 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  __shared__ int wide;
  __shared__ double total;
  if (threadIdx.x == 0) {
    total = __ldcg(reinterpret_cast<const double*>(acc_g));
    const int lo = 255 - static_cast<int>(__ldcg(reinterpret_cast<const unsigned int*>(acc_g + 1)));
    const int hi = static_cast<int>(__ldcg(reinterpret_cast<const unsigned int*>(acc_g + 2)));
    int lg = 0;  // ceil(log2 n)
    while ((int64_t{1} << lg) < nblocks) ++lg;
    wide = total > 0.0 && hi - lo + lg > 28;
    if (!wide) mean_out[0] = total > 0.0 ? round_div_f32(total, nblocks) : 0.f;
  }
  __syncthreads();
  if (!wide) return;
  // wide range: exact integer sums per exponent over all constants
  for (int i = threadIdx.x; i < 256; i += blockDim.x) sbins[i] = 0ull;
  __syncthreads();
  for (int64_t j = threadIdx.x; j < nblocks; j += blockDim.x) {
    const uint32_t u = __float_as_uint(__ldcg(absmax + j));
    const uint32_t e = u >> 23;
    const uint32_t sig = (u & 0x7FFFFFu) | (e ? 0x800000u : 0u);
    if (sig) atomicAdd(&sbins[e ? e : 1u], static_cast<unsigned long long>(sig));
  }
  __shared__ unsigned long long digit_sums[16];
  if (threadIdx.x < 16) digit_sums[threadIdx.x] = 0ull;
  __syncthreads();
  const float mean = exact_mean_f32(sbins, nblocks, digit_sums);
  if (threadIdx.x == 0) mean_out[0] = mean;
}

// Level 2: one warp per 256-block of constants, 8 constants per lane, centred on the
// mean that level 1 formed. Launched as the programmatic dependent of level 1.
// The E4M3 code of each y = fl32(cc / c1) comes from t8_nearest_codes2.
__global__ void __launch_bounds__(256)
    k_double_quantize(const float* __restrict__ absmax, int64_t nblocks,
                      const float* __restrict__ mean_in, const T8Thresholds th,
                      uint8_t* __restrict__ c2, float* __restrict__ c1) {
  __shared__ float sth[kT8Size - 1];
  for (int i = threadIdx.x; i < kT8Size - 1; i += blockDim.x) sth[i] = th.t[i];
  asm volatile("griddepcontrol.wait;" ::: "memory");  // level 1's absmax and mean
  __syncthreads();
  const float mean = __ldcg(mean_in);
  const int lane = threadIdx.x & 31;
  const int64_t ndq = (nblocks + 255) / 256;
  for (int64_t b = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32; b < ndq;
       b += static_cast<int64_t>(gridDim.x) * blockDim.x / 32) {
    const int64_t j0 = b * 256 + lane * 8;
    float cc[8];
    if (j0 + 8 <= nblocks) {  // two 16-byte loads (the absmax array is 256-byte aligned)
      const float4 a0 = reinterpret_cast<const float4*>(absmax + j0)[0];
      const float4 a1 = reinterpret_cast<const float4*>(absmax + j0)[1];
      cc[0] = a0.x; cc[1] = a0.y; cc[2] = a0.z; cc[3] = a0.w;
      cc[4] = a1.x; cc[5] = a1.y; cc[6] = a1.z; cc[7] = a1.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) cc[i] = (j0 + i < nblocks) ? absmax[j0 + i] : mean;
    }
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      cc[i] = __fsub_rn(cc[i], mean);  // 0 past the end
      m = fmaxf(m, fabsf(cc[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    // y = fl32(cc / c1): Markstein's correction step on one correctly rounded reciprocal
    // (as in level 1; exact for c1 >= 2^-64 wherever |y| > 2^-36, and every |y| below
    // that has the zero entry's code either way), plain IEEE division for smaller c1
    const bool fast = m >= 0x1p-64f;
    const float rc = fast ? __frcp_rn(m) : 0.f;
    auto quot = [&](float c) {
      if (fast) {
        const float q = __fmul_rn(c, rc);
        return __fmaf_rn(__fmaf_rn(-q, m, c), rc, q);
      }
      return m > 0.f ? __fdiv_rn(c, m) : 0.f;
    };
    uint32_t out[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; i += 2)
      out[i / 4] |= t8_nearest_codes2(quot(cc[i]), quot(cc[i + 1]), sth) << (8 * (i % 4));
    if (j0 + 8 <= nblocks) {
      reinterpret_cast<uint2*>(c2 + j0)[0] = make_uint2(out[0], out[1]);
    } else {
      for (int i = 0; i < 8 && j0 + i < nblocks; ++i)
        c2[j0 + i] = static_cast<uint8_t>(out[i / 4] >> (8 * (i % 4)));
    }
    if (lane == 0) c1[b] = m;
  }
}

// Standalone double dequantization: one thread per 8 codes (one 32-bit word), four words
// per thread and pass (kDqUnroll, a CTA's 256 threads apart so that every load and store
// instruction is coalesced), their loads all issued before the first is used.
constexpr int kDqUnroll = 4;
template <int CB>
__global__ void __launch_bounds__(256)
    k_dequant(const uint32_t* __restrict__ codes, const uint8_t* __restrict__ c2,
              const float* __restrict__ c1, const float* __restrict__ mean_p, int64_t nwords,
              uint4* __restrict__ out) {
  __shared__ float lut[16];
  __shared__ float t8[256];  // T8 by E4M3 code
  if (threadIdx.x < 16) lut[threadIdx.x] = code_level_rt<CB>(threadIdx.x);
  for (int e = threadIdx.x; e < 256; e += blockDim.x) t8[e] = t8_value(e);
  __syncthreads();
  const float mean = *mean_p;
  const int64_t chunk = static_cast<int64_t>(blockDim.x) * kDqUnroll;
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * chunk + threadIdx.x; base < nwords;
       base += static_cast<int64_t>(gridDim.x) * chunk) {
    uint32_t w[kDqUnroll], e[kDqUnroll];
    float g[kDqUnroll];
#pragma unroll
    for (int u = 0; u < kDqUnroll; ++u) {
      const int64_t i = base + u * static_cast<int64_t>(blockDim.x);
      if (i < nwords) {
        w[u] = __ldg(codes + i);
        e[u] = c2[i >> 3];   // 64-block of this word
        g[u] = c1[i >> 11];  // its 256-block of constants
      }
    }
#pragma unroll
    for (int u = 0; u < kDqUnroll; ++u) {
      const int64_t i = base + u * static_cast<int64_t>(blockDim.x);
      if (i < nwords) {
        const float s = block_scale_tab(t8, e[u], g[u], mean);
        uint32_t o[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const float a = __fmul_rn(lut[(w[u] >> (8 * p)) & 15u], s);
          const float b = __fmul_rn(lut[(w[u] >> (8 * p + 4)) & 15u], s);
          o[p] = pack_bf16x2_rn(a, b);
        }
        out[i] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
}

// CTAs of level 1: enough for every block, at most one resident wave (so that all of
// them run from the start) and at most kMaxQuantCtas.
template <typename T>
cudaError_t quant_ctas(int64_t nblocks, int* ctas) {
  static std::atomic<int> resident{0};  // CTAs per SM, looked up once per input type
  int per_sm = resident.load(std::memory_order_relaxed);
  if (per_sm == 0) {
    cudaError_t e =
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_quantize_blocks<T>, kQuantThreads, 0);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    resident.store(per_sm, std::memory_order_relaxed);
  }
  const int64_t per = kQuantThreads / kQuantLanes;  // blocks per CTA and pass
  const int64_t want = (nblocks + per - 1) / per;
  const int64_t wave = static_cast<int64_t>(num_sms()) * per_sm;
  const int64_t cap = wave < kMaxQuantCtas ? wave : kMaxQuantCtas;
  *ctas = static_cast<int>(want < cap ? (want < 1 ? 1 : want) : cap);
  return cudaSuccess;
}

}  // namespace

size_t quantize_workspace_bytes(int64_t n, int64_t k) {
  const int64_t nblocks = n * k / 64;
  return align_up(static_cast<size_t>(nblocks) * 4, 256) + 4 * sizeof(unsigned long long);
}

cudaError_t launch_quantize(const void* W, bool w_bf16, int64_t n, int64_t k, int codebook,
                            uint8_t* codes, uint8_t* c2, float* c1, float* mean, void* ws,
                            cudaStream_t st) {
  const int64_t nblocks = n * k / 64;
  float* absmax = static_cast<float*>(ws);
  unsigned long long* bins = reinterpret_cast<unsigned long long*>(
      static_cast<char*>(ws) + align_up(static_cast<size_t>(nblocks) * 4, 256));
  int ctas = 0;
  cudaError_t e = w_bf16 ? quant_ctas<uint16_t>(nblocks, &ctas) : quant_ctas<float>(nblocks, &ctas);
  if (e != cudaSuccess) return e;
  note_launches(3);  // clearing, blocks, then the double quantization
  {
    cudaLaunchConfig_t pc = {};
    pc.gridDim = dim3(1);
    pc.blockDim = dim3(32);
    pc.stream = st;
    cudaLaunchAttribute pa[1];
    pa[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pa[0].val.programmaticStreamSerializationAllowed = 1;
    pc.attrs = pa;
    pc.numAttrs = 1;
    e = cudaLaunchKernelEx(&pc, k_quantize_prep, bins);
    if (e != cudaSuccess) return e;
  }
  {
    cudaLaunchConfig_t c1cfg = {};
    c1cfg.gridDim = dim3(static_cast<unsigned>(ctas));
    c1cfg.blockDim = dim3(kQuantThreads);
    c1cfg.stream = st;
    cudaLaunchAttribute a1[1];
    a1[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a1[0].val.programmaticStreamSerializationAllowed = 1;
    c1cfg.attrs = a1;
    c1cfg.numAttrs = 1;
    const Nf4BucketTable& tab = code_buckets(codebook);
    e = w_bf16 ? cudaLaunchKernelEx(&c1cfg, k_quantize_blocks<uint16_t>,
                                    static_cast<const uint16_t*>(W), nblocks, tab, codes, absmax,
                                    bins, mean)
               : cudaLaunchKernelEx(&c1cfg, k_quantize_blocks<float>,
                                    static_cast<const float*>(W), nblocks, tab, codes, absmax,
                                    bins, mean);
    if (e != cudaSuccess) return e;
  }
  const int64_t ndq = (nblocks + 255) / 256;
  int64_t g = (ndq + 7) / 8;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  if (g > cap) g = cap;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(g));
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_double_quantize, static_cast<const float*>(absmax), nblocks,
                            static_cast<const float*>(mean), t8_thresholds(), c2, c1);
}

cudaError_t launch_dequant(const qlora_nf4_weight& w, uint16_t* out, cudaStream_t st) {
  const int64_t nwords = w.n_out * w.k_in / 8;
  auto kern = w.codebook == 1 ? k_dequant<1> : k_dequant<0>;
  static std::atomic<int> resident[kCodebooks];  // CTAs per SM, looked up once
  int per_sm = resident[w.codebook == 1].load(std::memory_order_relaxed);
  if (per_sm == 0) {
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, 0);
    if (e != cudaSuccess) return e;
    resident[w.codebook == 1].store(per_sm, std::memory_order_relaxed);
  }
  int64_t g = (nwords + 256 * kDqUnroll - 1) / (256 * kDqUnroll);
  const int64_t cap = static_cast<int64_t>(num_sms()) * (per_sm > 0 ? per_sm : 1);
  if (g > cap) g = cap;
  note_launches(1);
  kern<<<static_cast<int>(g), 256, 0, st>>>(reinterpret_cast<const uint32_t*>(w.codes), w.c2,
                                            w.c1, w.mean, nwords, reinterpret_cast<uint4*>(out));
  return cudaGetLastError();
}

}  // namespace qlora
