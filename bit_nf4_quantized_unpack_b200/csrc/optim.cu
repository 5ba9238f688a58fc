// optim.cu -- the optimizer step that follows the LoRA gradients: AdamW on the LoRA
// parameters with paged optimizer states in 32-bit or 8-bit form (page "QLoRA", itwiki.kr,
// section "페이지드 옵티마이저" (paged optimizers), and optim="paged_adamw_8bit" in the
// training example of section "계산 방식"). The states may live in unified memory
// (qlora_paged_alloc): the driver moves their pages to host memory when the GPU runs
// short and back when this kernel touches them, or ahead of it (qlora_paged_prefetch).
//
// Both kernels are HBM-bound streaming passes over the flat parameter buffer.
#include <cmath>

#include "internal.h"
#include "nf4_device.cuh"

namespace qlora {
namespace {

constexpr int kOptThreads = 256;  // 8 warps; a warp owns one 256-element state block
constexpr int kStateBlock = 256;  // elements per absmax block of an 8-bit state

struct AdamwConsts {
  float b1, b2, omb1, omb2, lr, eps, decay, bc1, bc2;
};

// One AdamW element. Every operation is one IEEE fp32 rounding, in this order, with no
// fused multiply-add:
//   m = b1 m' + (1-b1) g;  v = b2 v' + ((1-b2) g) g;  mh = m / bc1;  vh = v / bc2;
//   p = p (1 - lr wd) - lr (mh / (sqrt(vh) + eps)).
__device__ __forceinline__ float adamw_elem(float p, float g, float& m, float& v,
                                            const AdamwConsts& c) {
  m = __fadd_rn(__fmul_rn(c.b1, m), __fmul_rn(c.omb1, g));
  v = __fadd_rn(__fmul_rn(c.b2, v), __fmul_rn(__fmul_rn(c.omb2, g), g));
  const float mh = __fdiv_rn(m, c.bc1);
  const float vh = __fdiv_rn(v, c.bc2);
  const float u = __fdiv_rn(mh, __fadd_rn(__fsqrt_rn(vh), c.eps));
  return __fsub_rn(__fmul_rn(p, c.decay), __fmul_rn(c.lr, u));
}

// Eight consecutive fp32 values from element j0 (zeros past n). Plain loads: the
// parameter buffer is written by the same kernel, and the buffers may be managed memory.
__device__ __forceinline__ void load8(const float* src, int64_t j0, int64_t n, float (&v)[8]) {
  if (j0 + 8 <= n) {
    const float4 a = reinterpret_cast<const float4*>(src + j0)[0];
    const float4 b = reinterpret_cast<const float4*>(src + j0)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = (j0 + i < n) ? src[j0 + i] : 0.f;
  }
}

__device__ __forceinline__ void store8(float* dst, int64_t j0, int64_t n, const float (&v)[8]) {
  if (j0 + 8 <= n) {
    reinterpret_cast<float4*>(dst + j0)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(dst + j0)[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (j0 + i < n) dst[j0 + i] = v[i];
  }
}

// bf16 copy of eight parameters (the LoRA operand of the next forward).
__device__ __forceinline__ void store8_bf16(uint16_t* dst, int64_t j0, int64_t n, const float (&v)[8]) {
  if (j0 + 8 <= n) {
    reinterpret_cast<uint4*>(dst + j0)[0] =
        make_uint4(pack_bf16x2_rn(v[0], v[1]), pack_bf16x2_rn(v[2], v[3]),
                   pack_bf16x2_rn(v[4], v[5]), pack_bf16x2_rn(v[6], v[7]));
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (j0 + i < n) dst[j0 + i] = bf16_bits_rn(v[i]);
  }
}

__device__ __forceinline__ uint2 load_codes8(const uint8_t* src, int64_t j0, int64_t n) {
  if (j0 + 8 <= n) return reinterpret_cast<const uint2*>(src + j0)[0];
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (j0 + i < n) w[i / 4] |= static_cast<uint32_t>(src[j0 + i]) << (8 * (i % 4));
  return make_uint2(w[0], w[1]);
}

__device__ __forceinline__ void store_codes8(uint8_t* dst, int64_t j0, int64_t n, uint2 c) {
  if (j0 + 8 <= n) {
    reinterpret_cast<uint2*>(dst + j0)[0] = c;
  } else {
    const uint32_t w[2] = {c.x, c.y};
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (j0 + i < n) dst[j0 + i] = static_cast<uint8_t>(w[i / 4] >> (8 * (i % 4)));
  }
}

// y = fl32(x / d) for |x| <= d, or 0 when d = 0. With d >= 2^-64 and r = RN(1/d), one
// Markstein correction step (q = RN(x r), e = x - d q exact in an FMA, RN(q + e r)) gives
// the correctly rounded quotient for every |y| above 2^-36, far below the smallest T8
// decision threshold (about 2.2e-6), where the code is 0 either way; smaller d takes
// IEEE division.
__device__ __forceinline__ float block_ratio(float x, float d, float r) {
  if (r != 0.f) {
    const float q = __fmul_rn(x, r);
    return __fmaf_rn(__fmaf_rn(-q, d, x), r, q);
  }
  return d > 0.f ? __fdiv_rn(x, d) : 0.f;
}

// 8-bit states: per 256-element block one fp32 absmax and one E4M3 code per element;
// a stored value reads back as fl32(T8[code] * absmax). One warp per block, eight
// elements per lane; the new absmax is the warp's maximum of |m| (of v). Four CTAs per
// SM (64 registers): the step is bound by its dependent arithmetic, and more resident
// warps hide more of it.
constexpr int kOpt8CtasPerSm = 4;
__global__ void __launch_bounds__(kOptThreads, kOpt8CtasPerSm)
    k_adamw_8bit(float* __restrict__ p, uint16_t* __restrict__ p_bf16, const float* __restrict__ g,
                 int64_t n, uint8_t* __restrict__ mc, uint8_t* __restrict__ vc,
                 float* __restrict__ ma, float* __restrict__ va, const AdamwConsts c,
                 const T8Thresholds th) {
  __shared__ float sth[kT8Size - 1];
  __shared__ T8Search search;
  __shared__ float t8[256];  // T8 by E4M3 code
  for (int i = threadIdx.x; i < kT8Size - 1; i += blockDim.x) sth[i] = th.t[i];
  for (int e = threadIdx.x; e < 256; e += blockDim.x) t8[e] = t8_value(e);
  __syncthreads();
  build_t8_search(sth, search);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t nblk = (n + kStateBlock - 1) / kStateBlock;
  for (int64_t b = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32; b < nblk;
       b += static_cast<int64_t>(gridDim.x) * blockDim.x / 32) {
    const int64_t j0 = b * kStateBlock + lane * 8;
    float pv[8], gv[8], m[8], v[8];
    load8(p, j0, n, pv);
    load8(g, j0, n, gv);
    const uint2 mw = load_codes8(mc, j0, n), vw = load_codes8(vc, j0, n);
    const float am = ma[b], av = va[b];
    float mmax = 0.f, vmax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t mcode = ((i < 4 ? mw.x : mw.y) >> (8 * (i % 4))) & 0xFFu;
      const uint32_t vcode = ((i < 4 ? vw.x : vw.y) >> (8 * (i % 4))) & 0xFFu;
      m[i] = __fmul_rn(t8[mcode], am);
      v[i] = __fmul_rn(t8[vcode], av);
      pv[i] = adamw_elem(pv[i], gv[i], m[i], v[i], c);
      if (j0 + i >= n) m[i] = v[i] = 0.f;  // past the buffer: no part of the block maxima
      mmax = fmaxf(mmax, fabsf(m[i]));
      vmax = fmaxf(vmax, fabsf(v[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mmax = fmaxf(mmax, __shfl_xor_sync(0xFFFFFFFFu, mmax, o));
      vmax = fmaxf(vmax, __shfl_xor_sync(0xFFFFFFFFu, vmax, o));
    }
    uint32_t mo[2] = {0u, 0u}, vo[2] = {0u, 0u};
    const float rm = mmax >= 0x1p-64f ? __frcp_rn(mmax) : 0.f;  // warp-uniform choices
    const float rv = vmax >= 0x1p-64f ? __frcp_rn(vmax) : 0.f;
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const float ym0 = block_ratio(m[i], mmax, rm);
      const float ym1 = block_ratio(m[i + 1], mmax, rm);
      const float yv0 = block_ratio(v[i], vmax, rv);
      const float yv1 = block_ratio(v[i + 1], vmax, rv);
      mo[i / 4] |= t8_nearest_codes2(ym0, ym1, search) << (8 * (i % 4));
      vo[i / 4] |= t8_nearest_codes2(yv0, yv1, search) << (8 * (i % 4));
    }
    store8(p, j0, n, pv);
    if (p_bf16) store8_bf16(p_bf16, j0, n, pv);
    store_codes8(mc, j0, n, make_uint2(mo[0], mo[1]));
    store_codes8(vc, j0, n, make_uint2(vo[0], vo[1]));
    if (lane == 0) {
      ma[b] = mmax;
      va[b] = vmax;
    }
  }
}

// 32-bit states: m and v as fp32 arrays. Eight elements per thread.
__global__ void __launch_bounds__(kOptThreads)
    k_adamw_32bit(float* __restrict__ p, uint16_t* __restrict__ p_bf16, const float* __restrict__ g,
                  int64_t n, float* __restrict__ ms, float* __restrict__ vs, const AdamwConsts c) {
  const int64_t groups = (n + 7) / 8;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < groups;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t j0 = t * 8;
    float pv[8], gv[8], m[8], v[8];
    load8(p, j0, n, pv);
    load8(g, j0, n, gv);
    load8(ms, j0, n, m);
    load8(vs, j0, n, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) pv[i] = adamw_elem(pv[i], gv[i], m[i], v[i], c);
    store8(p, j0, n, pv);
    if (p_bf16) store8_bf16(p_bf16, j0, n, pv);
    store8(ms, j0, n, m);
    store8(vs, j0, n, v);
  }
}

}  // namespace

AdamwStateLayout adamw_state_layout(int64_t n, int state_bits) {
  AdamwStateLayout L{};
  if (state_bits == 8) {
    const int64_t nblk = (n + kStateBlock - 1) / kStateBlock;
    L.off_vc = align_up(static_cast<size_t>(n), 256);
    L.off_ma = L.off_vc + align_up(static_cast<size_t>(n), 256);
    L.off_va = L.off_ma + align_up(static_cast<size_t>(nblk) * 4, 256);
    L.total = L.off_va + align_up(static_cast<size_t>(nblk) * 4, 256);
  } else {
    L.off_vc = align_up(static_cast<size_t>(n) * 4, 256);  // v after m
    L.total = 2 * L.off_vc;
  }
  return L;
}

cudaError_t launch_adamw(float* p, uint16_t* p_bf16, const float* g, int64_t n, int state_bits,
                         void* state, const qlora_adamw_hparams& hp, cudaStream_t st) {
  // the fp32 constants of the step: (1 - b) and (1 - lr wd) in fp32, the bias corrections
  // 1 - b^t in fp64 rounded to fp32
  AdamwConsts c;
  c.b1 = hp.beta1;
  c.b2 = hp.beta2;
  c.omb1 = 1.0f - hp.beta1;
  c.omb2 = 1.0f - hp.beta2;
  c.lr = hp.lr;
  c.eps = hp.eps;
  volatile float lw = hp.lr * hp.weight_decay;  // rounded on its own, never fused
  c.decay = 1.0f - lw;
  c.bc1 = static_cast<float>(1.0 - std::pow(static_cast<double>(hp.beta1), static_cast<double>(hp.step)));
  c.bc2 = static_cast<float>(1.0 - std::pow(static_cast<double>(hp.beta2), static_cast<double>(hp.step)));
  const AdamwStateLayout L = adamw_state_layout(n, state_bits);
  uint8_t* base = static_cast<uint8_t*>(state);
  note_launches(1);
  if (state_bits == 8) {
    const int64_t nblk = (n + kStateBlock - 1) / kStateBlock;
    int64_t grid = (nblk + kOptThreads / 32 - 1) / (kOptThreads / 32);
    const int64_t cap = static_cast<int64_t>(num_sms()) * kOpt8CtasPerSm;  // one resident wave
    if (grid > cap) grid = cap;
    k_adamw_8bit<<<static_cast<unsigned>(grid), kOptThreads, 0, st>>>(
        p, p_bf16, g, n, base, base + L.off_vc, reinterpret_cast<float*>(base + L.off_ma),
        reinterpret_cast<float*>(base + L.off_va), c, t8_thresholds());
  } else {
    int64_t grid = ((n + 7) / 8 + kOptThreads - 1) / kOptThreads;
    const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
    if (grid > cap) grid = cap;
    k_adamw_32bit<<<static_cast<unsigned>(grid), kOptThreads, 0, st>>>(
        p, p_bf16, g, n, reinterpret_cast<float*>(base), reinterpret_cast<float*>(base + L.off_vc), c);
  }
  return cudaGetLastError();
}

}  // namespace qlora
