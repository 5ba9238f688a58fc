// codec.cu -- NF4 quantization with double-quantized constants, and the standalone
// double dequantization (page "QLoRA", itwiki.kr, sections "4비트 NormalFloat(NF4)" and
// "이중 양자화"). All three kernels are HBM-bound streaming passes.
#include <cuda_bf16.h>

#include "internal.h"
#include "nf4_device.cuh"

namespace qlora {
namespace {

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

// NF4 code of x in [-1, 1] from the bucket table in shared memory (entries: threshold,
// code as bits): bucket = round-half-even(512 x + 512), which the FMA leaves in the low
// mantissa bits of a number in [2^23, 2^24).
__device__ __forceinline__ uint32_t bucket_code(float x, const float2* sb) {
  const uint32_t idx =
      min(static_cast<uint32_t>(__float_as_int(__fmaf_rn(x, 512.0f, 12583424.0f)) - 0x4B400000),
          static_cast<uint32_t>(kCodeBuckets - 1));
  const float2 bk = sb[idx];
  return __float_as_uint(bk.y) + (x >= bk.x ? 1u : 0u);
}

// Level 1: one 64-block per group of 8 lanes (8 elements per lane). Writes the packed
// codes, the fp32 absmax of each block, and one fp64 partial sum of absmax per CTA.
//
// x = fl32(w / absmax) is computed with Markstein's correction step (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000 processor", IBM J.
// Res. Dev. 34, 1990): with r = RN(1/m), q = RN(w r) and e = w - m q (exact in an FMA),
// RN(q + e r) is the correctly rounded quotient. For m >= 2^-64, 1/m is finite and the
// residual stays exact for every |x| above 2^-36, far below the smallest threshold
// magnitude (0.04); blocks with a smaller absmax take plain IEEE division.
// The code of x comes from the 1025-bucket table (one shared-memory load and one compare).
template <typename T>
__global__ void __launch_bounds__(kQuantThreads)
    k_quantize_blocks(const T* __restrict__ W, int64_t nblocks,
                      const __grid_constant__ Nf4BucketTable tab, uint8_t* __restrict__ codes,
                      float* __restrict__ absmax, double* __restrict__ partial) {
  const int lane = threadIdx.x & 31;
  const int sub = lane & 7;
  const unsigned gmask = 0xFFu << (lane & 24);
  const int64_t per_cta = kQuantThreads / 8;
  __shared__ float2 sb[kCodeBuckets];  // (threshold, code as bits)
  for (int i = threadIdx.x; i < kCodeBuckets; i += blockDim.x)
    sb[i] = make_float2(tab.thr[i], __uint_as_float(static_cast<uint32_t>(tab.code[i])));
  __syncthreads();
  // the double quantization may be scheduled now; it waits for this grid's results
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  double acc = 0.0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * per_cta;
  int64_t b = blockIdx.x * per_cta + threadIdx.x / 8;
  // the next two blocks' elements are in flight while this one is coded
  Raw8<T> n0, n1;
  if (b < nblocks) n0.load(W + b * 64 + sub * 8);
  if (b + stride < nblocks) n1.load(W + (b + stride) * 64 + sub * 8);
  for (; b < nblocks; b += stride) {
    float v[8];
    n0.values(v);
    n0 = n1;
    if (b + 2 * stride < nblocks) n1.load(W + (b + 2 * stride) * 64 + sub * 8);
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[i]));
    m = fmaxf(m, __shfl_xor_sync(gmask, m, 1));
    m = fmaxf(m, __shfl_xor_sync(gmask, m, 2));
    m = fmaxf(m, __shfl_xor_sync(gmask, m, 4));
    uint32_t packed = 0;
    if (m >= 0x1p-64f) {
      const float r = __fdiv_rn(1.0f, m);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float w = v[i];
        const float q = __fmul_rn(w, r);
        const float e = __fmaf_rn(-q, m, w);
        packed |= bucket_code(__fmaf_rn(e, r, q), sb) << (4 * i);
      }
    } else {  // absmax zero or below 2^-64: plain IEEE division (x = 0 for a zero block)
#pragma unroll
      for (int i = 0; i < 8; ++i)
        packed |= bucket_code(m > 0.f ? __fdiv_rn(v[i], m) : 0.f, sb) << (4 * i);
    }
    reinterpret_cast<uint32_t*>(codes + b * 32)[sub] = packed;
    if (sub == 0) {
      absmax[b] = m;
      acc += static_cast<double>(m);
    }
  }
  __shared__ double red[kQuantThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  if (lane == 0) red[threadIdx.x / 32] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int i = 0; i < kQuantThreads / 32; ++i) s += red[i];
    partial[blockIdx.x] = s;
  }
}

// Index of entry i of T8 (ascending) -> its E4M3 bit pattern.
__device__ __forceinline__ uint32_t t8_index_to_code(int i) {
  return (i < 126) ? (0xFEu - static_cast<uint32_t>(i)) : (i == 126 ? 0u : static_cast<uint32_t>(i - 126));
}

// Level 2: the one mean of all block constants, then one warp per 256-block of constants,
// 8 constants per lane. Launched as the programmatic dependent of level 1: every CTA forms
// the mean itself from level 1's per-CTA fp64 partial sums, in the same order (fp64 sum,
// one rounding to fp32), and CTA 0 stores it.
__global__ void __launch_bounds__(256)
    k_double_quantize(const float* __restrict__ absmax, int64_t nblocks,
                      const double* __restrict__ partial, int nparts, float* __restrict__ mean_out,
                      const T8Thresholds th, uint8_t* __restrict__ c2, float* __restrict__ c1) {
  __shared__ float sth[kT8Size - 1];
  __shared__ double red[256 / 32];
  __shared__ float mean_s;
  for (int i = threadIdx.x; i < kT8Size - 1; i += blockDim.x) sth[i] = th.t[i];
  asm volatile("griddepcontrol.wait;" ::: "memory");  // level 1's absmax and partial sums
  {
    double acc = 0.0;
    for (int i = threadIdx.x; i < nparts; i += blockDim.x) acc += partial[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
      double sum = 0.0;
      for (int i = 0; i < 256 / 32; ++i) sum += red[i];
      mean_s = __double2float_rn(sum / static_cast<double>(nblocks));
      if (blockIdx.x == 0) mean_out[0] = mean_s;
    }
    __syncthreads();
  }
  const float mean = mean_s;
  const int lane = threadIdx.x & 31;
  const int64_t ndq = (nblocks + 255) / 256;
  for (int64_t b = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32; b < ndq;
       b += static_cast<int64_t>(gridDim.x) * blockDim.x / 32) {
    const int64_t j0 = b * 256 + lane * 8;
    float cc[8];
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      cc[i] = (j0 + i < nblocks) ? __fsub_rn(absmax[j0 + i], mean) : 0.f;
      m = fmaxf(m, fabsf(cc[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    uint32_t out[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float y = (m > 0.f) ? __fdiv_rn(cc[i], m) : 0.f;
      int pos = 0;  // number of thresholds <= y
#pragma unroll
      for (int step = 128; step >= 1; step >>= 1)
        if (pos + step <= kT8Size - 1 && sth[pos + step - 1] <= y) pos += step;
      out[i / 4] |= t8_index_to_code(pos) << (8 * (i % 4));
    }
    if (j0 + 8 <= nblocks) {
      reinterpret_cast<uint2*>(c2 + j0)[0] = make_uint2(out[0], out[1]);
    } else {
      for (int i = 0; i < 8 && j0 + i < nblocks; ++i)
        c2[j0 + i] = static_cast<uint8_t>(out[i / 4] >> (8 * (i % 4)));
    }
    if (lane == 0) c1[b] = m;
  }
}

// Standalone double dequantization: one thread per 8 codes (one 32-bit word).
template <int CB>
__global__ void __launch_bounds__(256)
    k_dequant(const uint32_t* __restrict__ codes, const uint8_t* __restrict__ c2,
              const float* __restrict__ c1, const float* __restrict__ mean_p, int64_t nwords,
              uint4* __restrict__ out) {
  __shared__ float lut[16];
  __shared__ float t8[256];  // T8 by E4M3 code
  if (threadIdx.x < 16) lut[threadIdx.x] = code_level<CB>(threadIdx.x);
  for (int e = threadIdx.x; e < 256; e += blockDim.x) t8[e] = t8_value(e);
  __syncthreads();
  const float mean = *mean_p;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nwords;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t j = i >> 3;  // 64-block of this word
    const float s = block_scale_tab(t8, c2[j], c1[j >> 8], mean);
    const uint32_t w = __ldg(codes + i);
    uint32_t o[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const float a = __fmul_rn(lut[(w >> (8 * p)) & 15u], s);
      const float b = __fmul_rn(lut[(w >> (8 * p + 4)) & 15u], s);
      o[p] = pack_bf16x2_rn(a, b);
    }
    out[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

int quant_ctas(int64_t nblocks) {
  const int64_t want = (nblocks + kQuantThreads / 8 - 1) / (kQuantThreads / 8);
  const int cap = num_sms() * 8 < kMaxQuantCtas ? num_sms() * 8 : kMaxQuantCtas;
  return static_cast<int>(want < cap ? (want < 1 ? 1 : want) : cap);
}

}  // namespace

size_t quantize_workspace_bytes(int64_t n, int64_t k) {
  const int64_t nblocks = n * k / 64;
  return align_up(static_cast<size_t>(nblocks) * 4, 256) + kMaxQuantCtas * sizeof(double);
}

cudaError_t launch_quantize(const void* W, bool w_bf16, int64_t n, int64_t k, int codebook,
                            uint8_t* codes, uint8_t* c2, float* c1, float* mean, void* ws,
                            cudaStream_t st) {
  const int64_t nblocks = n * k / 64;
  float* absmax = static_cast<float*>(ws);
  double* partial = reinterpret_cast<double*>(static_cast<char*>(ws) +
                                              align_up(static_cast<size_t>(nblocks) * 4, 256));
  const int ctas = quant_ctas(nblocks);
  note_launches(2);  // blocks, then the mean and double quantization
  if (w_bf16)
    k_quantize_blocks<uint16_t><<<ctas, kQuantThreads, 0, st>>>(
        static_cast<const uint16_t*>(W), nblocks, code_buckets(codebook), codes, absmax, partial);
  else
    k_quantize_blocks<float><<<ctas, kQuantThreads, 0, st>>>(
        static_cast<const float*>(W), nblocks, code_buckets(codebook), codes, absmax, partial);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
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
                            static_cast<const double*>(partial), ctas, mean, t8_thresholds(), c2,
                            c1);
}

cudaError_t launch_dequant(const qlora_nf4_weight& w, uint16_t* out, cudaStream_t st) {
  const int64_t nwords = w.n_out * w.k_in / 8;
  int64_t g = (nwords + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  if (g > cap) g = cap;
  auto kern = w.codebook == 1 ? k_dequant<1> : k_dequant<0>;
  note_launches(1);
  kern<<<static_cast<int>(g), 256, 0, st>>>(reinterpret_cast<const uint32_t*>(w.codes), w.c2,
                                            w.c1, w.mean, nwords, reinterpret_cast<uint4*>(out));
  return cudaGetLastError();
}

}  // namespace qlora
