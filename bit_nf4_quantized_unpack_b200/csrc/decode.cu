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

constexpr int kDecThreads = 128;
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
  int splits, units_per, nunits;  // K is cut into `splits` ranges of `units_per` 256-units
  int row_groups;                 // 32-row groups of W
  int t_groups;                   // 8-column groups of A (for T = X A)
  float* part;   // [splits][M][N]   partial sums of X W_hat^T
  float* tpart;  // [splits][M][r]   partial sums of T = X A
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

// Fragment mapping of the weight tasks: mma.m16n8k16 with the dequantized weight as the
// A operand (16 weight rows) and X as the B operand (8 token columns). Lane (g = lane/4,
// t = lane%4) owns K columns kb .. kb + 63 (kb = unit * 256 + 64 t) of weight rows g
// and g + 8 of each 16-row group; MMA number j (0..15) of a unit takes from every lane
// the four columns kb + 4j .. kb + 4j + 3: A pairs (rows g and g + 8), B pairs (token
// g). Summation order over K does not matter, so this relabelling of the MMA's k index
// is free, and the unpacked pairs land directly in the A operand registers.
constexpr int kGroups = 2;  // 16-row groups per warp (32 weight rows)

__device__ __forceinline__ int64_t lmin(int64_t x, int64_t y) { return x < y ? x : y; }

template <bool kTall>
__device__ __forceinline__ void decode_weight_task(const DecodeArgs& a, int rg, int split,
                                                   int lane, const float* t8) {
  const int g = lane >> 2, t = lane & 3;
  const int u0 = split * a.units_per;
  const int u1 = min(a.nunits, u0 + a.units_per);
  const int64_t K = a.K, N = a.N;
  const int64_t bpr = K / 64;
  const float mean = *a.mean;
  const int64_t rbase = static_cast<int64_t>(rg) * kRowsPerWarp;
  // token rows this lane feeds to the B operand; tokens >= M compute columns nobody stores
  const int64_t xr0 = lmin(g, a.M - 1);
  const int64_t xr1 = lmin(g + 8, a.M - 1);
  float acc[kGroups][kTall ? 2 : 1][4];
#pragma unroll
  for (int q = 0; q < kGroups; ++q)
#pragma unroll
    for (int h = 0; h < (kTall ? 2 : 1); ++h)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[q][h][i] = 0.f;

  for (int u = u0; u < u1; ++u) {
    const int64_t kraw = static_cast<int64_t>(u) * kUnitK + 64 * t;
    const bool kv = kraw < K;
    const int64_t kb = kv ? kraw : K - 64;  // clamped: the scale below is zero then
    // every load of this unit is issued before any math; rows beyond N are clamped and
    // get a zero scale
    uint4 cq[kGroups][2][2];
    uint32_t e2[kGroups][2];
    float e1[kGroups][2];
#pragma unroll
    for (int q = 0; q < kGroups; ++q)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t row = lmin(rbase + q * 16 + g + 8 * h, N - 1);
        const uint8_t* p = a.codes + row * (K / 2) + kb / 2;
        cq[q][h][0] = ldg_stream(p);
        cq[q][h][1] = ldg_stream(p + 16);
        const int64_t j = row * bpr + kb / 64;
        e2[q][h] = __ldg(a.c2 + j);
        e1[q][h] = __ldg(a.c1 + (j >> 8));
      }
    uint32_t xa[32], xb[32];
    load_x64(a.X, K, xr0, true, kb, xa);
    if (kTall) load_x64(a.X, K, xr1, true, kb, xb);
#pragma unroll
    for (int q = 0; q < kGroups; ++q) {
      Nf4Lut lut[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const bool live = kv && (rbase + q * 16 + g + 8 * h) < N;
        build_lut(live ? block_scale_tab(t8, e2[q][h], e1[q][h], mean) : 0.f, lut[h]);
      }
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        uint32_t o0[4], o1[4];
        lut_decode8(w < 4 ? (&cq[q][0][0].x)[w] : (&cq[q][0][1].x)[w - 4], lut[0], o0);
        lut_decode8(w < 4 ? (&cq[q][1][0].x)[w] : (&cq[q][1][1].x)[w - 4], lut[1], o1);
        mma_bf16_16816(acc[q][0], o0[0], o1[0], o0[1], o1[1], xa[4 * w], xa[4 * w + 1]);
        mma_bf16_16816(acc[q][0], o0[2], o1[2], o0[3], o1[3], xa[4 * w + 2], xa[4 * w + 3]);
        if (kTall) {
          mma_bf16_16816(acc[q][kTall ? 1 : 0], o0[0], o1[0], o0[1], o1[1], xb[4 * w],
                         xb[4 * w + 1]);
          mma_bf16_16816(acc[q][kTall ? 1 : 0], o0[2], o1[2], o0[3], o1[3], xb[4 * w + 2],
                         xb[4 * w + 3]);
        }
      }
    }
  }
  // C fragment: c0,c1 = (weight row g, tokens 2t, 2t+1), c2,c3 = (row g + 8, same tokens);
  // the second accumulator (M > 8) holds tokens 8 + 2t, 8 + 2t + 1.
#pragma unroll
  for (int q = 0; q < kGroups; ++q)
#pragma unroll
    for (int hm = 0; hm < (kTall ? 2 : 1); ++hm)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int64_t row = rbase + q * 16 + g + 8 * (i >> 1);
        const int64_t m = 8 * hm + 2 * t + (i & 1);
        if (row < N && m < a.M)
          a.part[(static_cast<int64_t>(split) * a.M + m) * N + row] = acc[q][hm][i];
      }
}

// T partials over the K range of `split` for A columns tg*8 .. tg*8+7 (A [K, r] plays
// the weight: its column is gathered with strided bf16 loads).
template <bool kTall>
__device__ __forceinline__ void decode_t_task(const DecodeArgs& a, int idx, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const int tg = idx % a.t_groups;
  const int split = idx / a.t_groups;
  const int u0 = split * a.units_per;
  const int u1 = min(a.nunits, u0 + a.units_per);
  const int col = tg * 8 + g;
  float d[4] = {0.f, 0.f, 0.f, 0.f};
  for (int u = u0; u < u1; ++u) {
    const int64_t kb = static_cast<int64_t>(u) * kUnitK + 64 * t;
    const bool kv = kb < a.K;
    const bool live = kv && col < a.r;
    uint32_t bw[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      uint32_t lo = 0, hi = 0;
      if (live) {
        lo = __ldg(a.A + (kb + 2 * i) * a.r + col);
        hi = __ldg(a.A + (kb + 2 * i + 1) * a.r + col);
      }
      bw[i] = lo | (hi << 16);
    }
    uint32_t xa[32], xb[32];
    load_x64(a.X, a.K, g, kv && g < a.M, kb, xa);
    if (kTall) load_x64(a.X, a.K, g + 8, kv && g + 8 < a.M, kb, xb);
#pragma unroll
    for (int j = 0; j < 16; ++j)
      mma_bf16_16816(d, xa[2 * j], kTall ? xb[2 * j] : 0u, xa[2 * j + 1],
                     kTall ? xb[2 * j + 1] : 0u, bw[2 * j], bw[2 * j + 1]);
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int64_t m = g + 8 * h;
    if (m >= a.M) continue;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int c = tg * 8 + 2 * t + e;
      if (c < a.r) a.tpart[(static_cast<int64_t>(split) * a.M + m) * a.r + c] = d[2 * h + e];
    }
  }
}

template <bool kTall>  // kTall: M > 8 (tokens 8..15 live in the upper fragment rows)
__global__ void __launch_bounds__(kDecThreads, kTall ? 2 : 3) k_decode_gemv(const DecodeArgs a) {
  // the finalize kernel may be scheduled now; it waits for this grid's results
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ float t8[256];  // T8 by E4M3 code
  for (int i = threadIdx.x; i < 256; i += blockDim.x) t8[i] = t8_value(i);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int task = blockIdx.x * (kDecThreads / 32) + warp;
  const int wtasks = a.row_groups * a.splits;
  if (task < wtasks)
    decode_weight_task<kTall>(a, task % a.row_groups, task / a.row_groups, lane, t8);
  else if (task < wtasks + a.t_groups * a.splits)
    decode_t_task<kTall>(a, task - wtasks, lane);
}

// One CTA per 32 output columns: T = sum of its split partials (lanes over splits,
// warp shuffles), the Y partials summed by 8 groups of splits then combined through
// shared memory, plus scale * T B, rounded to bf16.
constexpr int kFinCols = 32;
__global__ void __launch_bounds__(256)
    k_decode_finalize(const float* __restrict__ part, const float* __restrict__ tpart,
                      int splits, int64_t M, int64_t N, int r, float scale,
                      const uint16_t* __restrict__ B, uint16_t* __restrict__ Y,
                      float* __restrict__ T_save) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the GEMV's partial sums are complete
  __shared__ float T[16 * 64];
  __shared__ float red[8][16][kFinCols];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mr = static_cast<int>(M) * r;
  for (int e = warp; e < mr; e += 8) {
    float v = 0.f;
    for (int s = lane; s < splits; s += 32) v += tpart[static_cast<int64_t>(s) * mr + e];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    if (lane == 0) {
      T[e] = v;
      if (T_save && blockIdx.x == 0) T_save[e] = v;
    }
  }
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kFinCols;
  const int64_t n = n0 + lane;
  float acc[16];
#pragma unroll
  for (int m = 0; m < 16; ++m) acc[m] = 0.f;
  if (n < N) {
    for (int s = warp; s < splits; s += 8) {
#pragma unroll
      for (int m = 0; m < 16; ++m)
        if (m < M) acc[m] += part[(static_cast<int64_t>(s) * M + m) * N + n];
    }
  }
#pragma unroll
  for (int m = 0; m < 16; ++m)
    if (m < M) red[warp][m][lane] = acc[m];
  __syncthreads();
  for (int idx = threadIdx.x; idx < static_cast<int>(M) * kFinCols; idx += blockDim.x) {
    const int m = idx / kFinCols, c = idx % kFinCols;
    const int64_t nn = n0 + c;
    if (nn >= N) continue;
    float y = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) y += red[w][m][c];
    float lora = 0.f;
    for (int j = 0; j < r; ++j)
      lora += T[m * r + j] * __uint_as_float(static_cast<uint32_t>(__ldg(B + j * N + nn)) << 16);
    Y[m * N + nn] = bf16_bits_rn(y + scale * lora);
  }
}

struct DecodePlan {
  int splits, units_per, nunits, row_groups, t_groups;
};

DecodePlan plan_decode(const LinearShape& s) {
  DecodePlan p;
  p.nunits = static_cast<int>((s.K + kUnitK - 1) / kUnitK);
  p.row_groups = static_cast<int>((s.N + kRowsPerWarp - 1) / kRowsPerWarp);
  p.t_groups = (s.r + 7) / 8;
  // As many K splits as keep the fp32 partial sums (splits * M * N * 4 bytes) to a few
  // percent of the weight bytes (N * K / 2): splits <= K / (128 M).
  int64_t want = std::max<int64_t>(1, s.K / (128 * std::max<int64_t>(1, s.M)));
  want = std::min<int64_t>(want, p.nunits);
  p.units_per = static_cast<int>((p.nunits + want - 1) / want);
  p.splits = (p.nunits + p.units_per - 1) / p.units_per;
  return p;
}

size_t part_bytes(const DecodePlan& p, const LinearShape& s) {
  return align_up(static_cast<size_t>(p.splits) * s.M * s.N * 4, 256);
}
size_t tpart_bytes(const DecodePlan& p, const LinearShape& s) {
  return align_up(static_cast<size_t>(p.splits) * s.M * s.r * 4, 256);
}

// The GEMV grid, then the finalize kernel with programmatic dependent launch.
qlora_status launch_decode(const uint16_t* X, const qlora_nf4_weight& w, const uint16_t* A,
                           const uint16_t* B, const LinearShape& s, const DecodePlan& p,
                           uint16_t* Y, float* T_save, char* scratch, cudaStream_t st) {
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
  a.part = reinterpret_cast<float*>(scratch);
  a.tpart = reinterpret_cast<float*>(scratch + part_bytes(p, s));
  const int64_t warps = static_cast<int64_t>(p.row_groups + p.t_groups) * p.splits;
  const unsigned ctas = static_cast<unsigned>((warps + kDecThreads / 32 - 1) / (kDecThreads / 32));
  if (s.M > 8)
    k_decode_gemv<true><<<ctas, kDecThreads, 0, st>>>(a);
  else
    k_decode_gemv<false><<<ctas, kDecThreads, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((s.N + kFinCols - 1) / kFinCols));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, k_decode_finalize, static_cast<const float*>(a.part),
                         static_cast<const float*>(a.tpart), p.splits, s.M, s.N, s.r, s.scale, B,
                         Y, T_save);
  if (e != cudaSuccess) return cuda_status(e);
  return QLORA_OK;
}

}  // namespace

size_t decode_workspace(const LinearShape& s) {
  const DecodePlan p = plan_decode(s);
  return part_bytes(p, s) + tpart_bytes(p, s) + 256;
}

qlora_status decode_forward(const uint16_t* X, const qlora_nf4_weight& w, const uint16_t* A,
                            const uint16_t* B, const LinearShape& s, uint16_t* Y,
                            float* T_save, void* ws, cudaStream_t st) {
  return launch_decode(X, w, A, B, s, plan_decode(s), Y, T_save, static_cast<char*>(ws), st);
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
  // Fewer K splits when the planned partial sums do not fit the static array.
  const size_t per_split = static_cast<size_t>(M) * s.N * 4;
  const size_t fixed = tpart_bytes(p, s) + 512;
  const size_t fit = fixed < kStaticScratchBytes ? (kStaticScratchBytes - fixed) / per_split : 0;
  if (fit < 1) {
    char msg[200];
    std::snprintf(msg, sizeof(msg),
                  "qlora_linear_fwd_decode_static: needs more than %zu bytes of partial sums; "
                  "the static scratch holds %zu bytes",
                  per_split + fixed, kStaticScratchBytes);
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
  // Every partial sum the finalize kernel reads is written by the GEMV first, so
  // nothing left in the array by an earlier call needs clearing.
  return launch_decode(X, w, A, B, s, p, Y, T_save, static_cast<char*>(scratch),
                       static_cast<cudaStream_t>(stream));
}

