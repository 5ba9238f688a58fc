// decode.cu -- the QLoRA linear forward for M <= 16 tokens (decode), which is bound by
// the HBM read of the packed weight (0.516 B per parameter).
//
//   Y = bf16(X W_hat^T + scale (X A) B)    (page "QLoRA", itwiki.kr, section "계산 방식";
//                                           alpha/r from page "quantization", minnong511)
//
// k_decode_gemv: each warp owns 32 weight rows and a contiguous range of K. Lanes load
// 32 bytes of packed codes of one row with 128-bit loads, double-dequantize them in
// registers (16-entry bf16 table per 64-block, prmt lookups) straight into the B
// fragments of mma.m16n8k16 (X is the A operand, tokens padded to 16 rows). The
// dequantized weight never leaves registers. Extra warps compute the split partial
// sums of T = X A the same way (A plays the weight). Partial sums go to a workspace.
// k_decode_finalize: sums the K splits, adds scale * T B and rounds to bf16.
//
// On tensor cores the multiply-adds cost nothing next to the unpack; mma.sync takes its
// operands from registers, which is exactly where the unpack leaves the weights.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdio>
#include <mutex>

#include "internal.h"
#include "nf4_device.cuh"

namespace qlora {
namespace {

constexpr int kDecThreads = 256;
constexpr int kRowsPerWarp = 32;
constexpr int kUnitK = 256;  // K covered by one warp step (4 lanes x 64)

struct DecodeArgs {
  const uint8_t* codes;
  const uint8_t* c2;
  const float* c1;
  const float* mean;
  const uint16_t* X;
  const uint16_t* A;
  int64_t M, N, K;
  int r;
  int splits, units_per, nunits;
  int row_groups, t_groups;
  float* part;   // [splits][M][N]
  float* tpart;  // [splits][M][r]
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// 64 consecutive bf16 of X row `row` starting at column k, as 32 packed pairs (zeros
// when the row is padding).
__device__ __forceinline__ void load_x64(const uint16_t* X, int64_t K, int64_t row, bool live,
                                         int64_t k, uint32_t (&x)[32]) {
  if (live) {
    const uint4* p = reinterpret_cast<const uint4*>(X + row * K + k);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint4 v = __ldg(p + i);
      x[4 * i] = v.x;
      x[4 * i + 1] = v.y;
      x[4 * i + 2] = v.z;
      x[4 * i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) x[i] = 0u;
  }
}

template <bool kTall>  // kTall: M > 8 (tokens 8..15 live in the upper fragment rows)
__global__ void __launch_bounds__(kDecThreads, kTall ? 1 : 2) k_decode_gemv(const DecodeArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int task = blockIdx.x * (kDecThreads / 32) + warp;
  const int ngroups = a.row_groups + a.t_groups;
  if (task >= ngroups * a.splits) return;
  const int group = task % ngroups;
  const int split = task / ngroups;
  const bool is_t = group >= a.row_groups;
  const int g = lane >> 2, t = lane & 3;
  const int u0 = split * a.units_per;
  const int u1 = min(a.nunits, u0 + a.units_per);
  const int64_t bpr = a.K / 64;
  const float mean = *a.mean;
  const int64_t rbase = static_cast<int64_t>(is_t ? group - a.row_groups : group) * kRowsPerWarp;
  const int64_t rlimit = is_t ? a.r : a.N;

  float acc[4][4];
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[q][i] = 0.f;

  for (int u = u0; u < u1; ++u) {
    const int64_t kb = static_cast<int64_t>(u) * kUnitK + 64 * t;
    const bool kv = kb < a.K;
    if (!is_t) {
      uint32_t xa[32], xb[32];
      load_x64(a.X, a.K, g, kv && g < a.M, kb, xa);
      if (kTall) load_x64(a.X, a.K, g + 8, kv && g + 8 < a.M, kb, xb);
      // issue the code and constant loads of all four row groups before any math
      uint4 cq[4][2];
      uint32_t e2[4];
      float e1[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int64_t row = rbase + q * 8 + g;
        cq[q][0] = cq[q][1] = make_uint4(0, 0, 0, 0);
        e2[q] = 0u;
        e1[q] = 0.f;
        if (kv && row < rlimit) {
          const uint8_t* p = a.codes + row * (a.K / 2) + kb / 2;
          cq[q][0] = ldg_stream(p);
          cq[q][1] = ldg_stream(p + 16);
          const int64_t j = row * bpr + kb / 64;
          e2[q] = __ldg(a.c2 + j);
          e1[q] = __ldg(a.c1 + (j >> 8));
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (rbase + q * 8 >= rlimit) continue;  // warp-uniform
        const int64_t row = rbase + q * 8 + g;
        const float sc = (kv && row < rlimit) ? block_scale(e2[q], e1[q], mean) : 0.f;
        Nf4Lut lut;
        build_lut(sc, lut);
        const uint32_t words[8] = {cq[q][0].x, cq[q][0].y, cq[q][0].z, cq[q][0].w,
                                   cq[q][1].x, cq[q][1].y, cq[q][1].z, cq[q][1].w};
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          uint32_t o[4];
          lut_decode8(words[w], lut, o);
          mma_bf16_16816(acc[q], xa[4 * w], kTall ? xb[4 * w] : 0u,
                         xa[4 * w + 1], kTall ? xb[4 * w + 1] : 0u, o[0],
                         o[1]);
          mma_bf16_16816(acc[q], xa[4 * w + 2], kTall ? xb[4 * w + 2] : 0u,
                         xa[4 * w + 3], kTall ? xb[4 * w + 3] : 0u, o[2],
                         o[3]);
        }
      }
    } else {
      // A [K, r] column `row` plays the weight: strided bf16 loads, pairs along k
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        if (rbase + q * 8 >= rlimit) continue;  // warp-uniform
        const int64_t row = rbase + q * 8 + g;
        const bool live = kv && row < rlimit;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
        for (int j = 0; j < 16; ++j) {
          uint32_t b[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t lo = 0, hi = 0;
            if (live) {
              lo = __ldg(a.A + (kb + 4 * j + 2 * h) * a.r + row);
              hi = __ldg(a.A + (kb + 4 * j + 2 * h + 1) * a.r + row);
            }
            b[h] = lo | (hi << 16);
          }
          // the X pairs of this k group, re-read from L1 to keep registers free
          const uint32_t* xr = reinterpret_cast<const uint32_t*>(a.X + g * a.K + kb + 4 * j);
          const uint32_t* xr8 = reinterpret_cast<const uint32_t*>(a.X + (g + 8) * a.K + kb + 4 * j);
          const bool lg = kv && g < a.M, lg8 = kv && g + 8 < a.M;
          mma_bf16_16816(d, lg ? __ldg(xr) : 0u, lg8 ? __ldg(xr8) : 0u, lg ? __ldg(xr + 1) : 0u,
                         lg8 ? __ldg(xr8 + 1) : 0u, b[0], b[1]);
        }
#pragma unroll
        for (int qq = 0; qq < 4; ++qq)
          if (qq == q)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[qq][i] += d[i];
      }
    }
  }
  // C fragment: acc[q][0..1] = (token g, rows 2t, 2t+1), acc[q][2..3] = (token g+8, ...)
#pragma unroll
  for (int q = 0; q < 4; ++q) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t m = g + 8 * h;
      if (m >= a.M) continue;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int64_t row = rbase + q * 8 + 2 * t + e;
        if (row >= rlimit) continue;
        if (is_t)
          a.tpart[(static_cast<int64_t>(split) * a.M + m) * a.r + row] = acc[q][2 * h + e];
        else
          a.part[(static_cast<int64_t>(split) * a.M + m) * a.N + row] = acc[q][2 * h + e];
      }
    }
  }
}

__global__ void __launch_bounds__(256)
    k_decode_finalize(const float* __restrict__ part, const float* __restrict__ tpart,
                      int splits, int64_t M, int64_t N, int r, float scale,
                      const uint16_t* __restrict__ B, uint16_t* __restrict__ Y,
                      float* __restrict__ T_save) {
  __shared__ float T[16 * 64];
  for (int i = threadIdx.x; i < M * r; i += blockDim.x) {
    float v = 0.f;
    for (int s = 0; s < splits; ++s) v += tpart[static_cast<int64_t>(s) * M * r + i];
    T[i] = v;
    if (T_save && blockIdx.x == 0) T_save[i] = v;
  }
  __syncthreads();
  const int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (n >= N) return;
  float lora[16];
#pragma unroll
  for (int m = 0; m < 16; ++m) lora[m] = 0.f;
  for (int j = 0; j < r; ++j) {
    const float bj = __uint_as_float(static_cast<uint32_t>(__ldg(B + j * N + n)) << 16);
#pragma unroll
    for (int m = 0; m < 16; ++m)
      if (m < M) lora[m] += T[m * r + j] * bj;
  }
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    if (m >= M) break;
    float y = 0.f;
    for (int s = 0; s < splits; ++s) y += part[(static_cast<int64_t>(s) * M + m) * N + n];
    Y[m * N + n] = bf16_bits_rn(y + scale * lora[m]);
  }
}

struct DecodePlan {
  int splits, units_per, nunits, row_groups, t_groups;
};

DecodePlan plan_decode(const LinearShape& s) {
  DecodePlan p;
  p.nunits = static_cast<int>((s.K + kUnitK - 1) / kUnitK);
  p.row_groups = static_cast<int>((s.N + kRowsPerWarp - 1) / kRowsPerWarp);
  p.t_groups = (s.r + kRowsPerWarp - 1) / kRowsPerWarp;
  const int64_t target_warps = static_cast<int64_t>(num_sms()) * 16;
  int64_t want = (target_warps + p.row_groups - 1) / p.row_groups;
  // keep the fp32 partials small next to the weight bytes
  want = std::min<int64_t>(want, std::max<int64_t>(1, s.K / (64 * std::max<int64_t>(1, s.M))));
  want = std::max<int64_t>(1, std::min<int64_t>(want, p.nunits));
  p.units_per = static_cast<int>((p.nunits + want - 1) / want);
  p.splits = (p.nunits + p.units_per - 1) / p.units_per;
  return p;
}

}  // namespace

size_t decode_workspace(const LinearShape& s) {
  const DecodePlan p = plan_decode(s);
  return align_up(static_cast<size_t>(p.splits) * s.M * s.N * 4, 256) +
         align_up(static_cast<size_t>(p.splits) * s.M * s.r * 4, 256) + 256;
}

qlora_status decode_forward(const uint16_t* X, const qlora_nf4_weight& w, const uint16_t* A,
                            const uint16_t* B, const LinearShape& s, uint16_t* Y,
                            float* T_save, void* ws, cudaStream_t st) {
  const DecodePlan p = plan_decode(s);
  DecodeArgs a;
  a.codes = w.codes;
  a.c2 = w.c2;
  a.c1 = w.c1;
  a.mean = w.mean;
  a.X = X;
  a.A = A;
  a.M = s.M;
  a.N = s.N;
  a.K = s.K;
  a.r = s.r;
  a.splits = p.splits;
  a.units_per = p.units_per;
  a.nunits = p.nunits;
  a.row_groups = p.row_groups;
  a.t_groups = p.t_groups;
  char* base = static_cast<char*>(ws);
  a.part = reinterpret_cast<float*>(base);
  a.tpart = reinterpret_cast<float*>(
      base + align_up(static_cast<size_t>(p.splits) * s.M * s.N * 4, 256));
  const int64_t warps = static_cast<int64_t>(p.row_groups + p.t_groups) * p.splits;
  const unsigned ctas = static_cast<unsigned>((warps + 7) / 8);
  if (s.M > 8)
    k_decode_gemv<true><<<ctas, kDecThreads, 0, st>>>(a);
  else
    k_decode_gemv<false><<<ctas, kDecThreads, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e);
  k_decode_finalize<<<static_cast<unsigned>((s.N + 255) / 256), 256, 0, st>>>(
      a.part, a.tpart, p.splits, s.M, s.N, s.r, s.scale, B, Y, T_save);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e);
  return QLORA_OK;
}

}  // namespace qlora

// ============================================================================
// Allocation-free variant of the decode forward.
//
// Some callers cannot call cudaMalloc when they run the layer: a runtime that plans
// all device memory once at start-up and forbids later allocation, or a decode loop
// that must not pay cudaMalloc's implicit device synchronisation on every token.
// They cannot hand over a workspace either. For them, qlora_linear_fwd_decode_static
// keeps the split partial sums in the fixed array below, which every GPU that loads
// this library holds until the process exits.
namespace qlora {
namespace {

constexpr size_t kStaticScratchBytes = size_t{4} << 20;  // 4 MiB per device
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

constexpr int kMaxScratchDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxScratchDevices] = {};

// Device address of g_decode_scratch on the current device. In host code the name
// g_decode_scratch is only a host-side stand-in, so the address is looked up once
// per device with that device current, and cached.
qlora_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  if (dev < 0 || dev >= kMaxScratchDevices) {
    set_last_error("device index out of range for the static scratch table");
    return QLORA_ERR_INVALID_ARG;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return cuda_status(e);
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return QLORA_OK;
}

bool aligned16_ptr(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

}  // namespace qlora

extern "C" qlora_status qlora_linear_fwd_decode_static(const uint16_t* X, int64_t M,
                                                       qlora_nf4_weight w, const uint16_t* A,
                                                       const uint16_t* B, int r, float scale,
                                                       uint16_t* Y, float* T_save, void* stream) {
  using namespace qlora;
  if (!w.codes || !w.c2 || !w.c1 || !w.mean) return QLORA_ERR_INVALID_ARG;
  if (w.n_out < 1 || w.k_in < 64 || w.k_in % 64 != 0 || w.n_out % 8 != 0 ||
      w.n_out > (int64_t{1} << 31) || w.k_in > (int64_t{1} << 31))
    return QLORA_ERR_SHAPE;
  if (M < 0 || M > kDecodeMaxM) {
    set_last_error("qlora_linear_fwd_decode_static serves 0 <= M <= 16 tokens");
    return QLORA_ERR_SHAPE;
  }
  if (r < 8 || r > 64 || r % 8 != 0) return QLORA_ERR_INVALID_ARG;
  if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f) return QLORA_ERR_INVALID_ARG;
  if (!aligned16_ptr(w.codes) || !aligned16_ptr(w.c2) || !aligned16_ptr(w.c1) ||
      !aligned16_ptr(w.mean))
    return QLORA_ERR_ALIGN;
  if (M == 0) return QLORA_OK;
  if (!X || !A || !B || !Y) return QLORA_ERR_INVALID_ARG;
  if (!aligned16_ptr(X) || !aligned16_ptr(A) || !aligned16_ptr(B) || !aligned16_ptr(Y) ||
      (T_save && !aligned16_ptr(T_save)))
    return QLORA_ERR_ALIGN;

  const LinearShape s{M, w.n_out, w.k_in, r, scale};
  DecodePlan p = plan_decode(s);
  // Fewer K splits when the planned partial sums would not fit the static array.
  const size_t per_split = static_cast<size_t>(M) * (s.N + s.r) * 4;
  const size_t fit = (kStaticScratchBytes - 512) / per_split;
  if (fit < 1) {
    char msg[200];
    std::snprintf(msg, sizeof(msg),
                  "qlora_linear_fwd_decode_static: M * (N + r) * 4 = %zu bytes exceeds the "
                  "%zu-byte static scratch",
                  per_split, kStaticScratchBytes);
    set_last_error(msg);
    return QLORA_ERR_WORKSPACE;
  }
  if (static_cast<size_t>(p.splits) > fit) {
    p.units_per = static_cast<int>((p.nunits + fit - 1) / fit);
    p.splits = (p.nunits + p.units_per - 1) / p.units_per;
  }
  void* scratch = nullptr;
  qlora_status q = scratch_address(&scratch);
  if (q != QLORA_OK) return q;

  DecodeArgs a;
  a.codes = w.codes;
  a.c2 = w.c2;
  a.c1 = w.c1;
  a.mean = w.mean;
  a.X = X;
  a.A = A;
  a.M = s.M;
  a.N = s.N;
  a.K = s.K;
  a.r = s.r;
  a.splits = p.splits;
  a.units_per = p.units_per;
  a.nunits = p.nunits;
  a.row_groups = p.row_groups;
  a.t_groups = p.t_groups;
  // Every partial sum below is written by the GEMV before the finalize kernel reads
  // it, so nothing left in the array by an earlier call needs clearing.
  char* base = static_cast<char*>(scratch);
  a.part = reinterpret_cast<float*>(base);
  a.tpart = reinterpret_cast<float*>(
      base + align_up(static_cast<size_t>(p.splits) * s.M * s.N * 4, 256));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t warps = static_cast<int64_t>(p.row_groups + p.t_groups) * p.splits;
  const unsigned ctas = static_cast<unsigned>((warps + 7) / 8);
  if (s.M > 8)
    k_decode_gemv<true><<<ctas, kDecThreads, 0, st>>>(a);
  else
    k_decode_gemv<false><<<ctas, kDecThreads, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e);
  k_decode_finalize<<<static_cast<unsigned>((s.N + 255) / 256), 256, 0, st>>>(
      a.part, a.tpart, p.splits, s.M, s.N, s.r, s.scale, B, Y, T_save);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e);
  return QLORA_OK;
}

