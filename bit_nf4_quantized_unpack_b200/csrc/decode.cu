// decode.cu -- the QLoRA linear forward for M <= 16 tokens (decode), which is bound by
// reading the packed weight (0.516 B per parameter) and by the integer work of
// expanding it.
//
//   Y = bf16(X W_hat^T + scale (X A) B)    (page "QLoRA", itwiki.kr, section "계산 방식";
//                                           alpha/r from page "quantization", minnong511)
//
// k_decode_lora_down: T = X A on one cluster of 8 CTAs that split K; the CTA partial sums
//   meet through distributed shared memory. It also clears the GEMV's arrival counters.
// k_decode_gemv: each warp owns 16 (M <= 8) or 32 weight rows and a range of K. Lanes load
//   32 bytes of packed codes of one row with 128-bit loads (the next 256-wide unit while
//   the current one is expanded), double-dequantize them in registers (16-entry bf16
//   table per 64-block, prmt lookups) straight into the A fragments of mma.m16n8k16 (X is
//   the B operand). The dequantized weight never leaves registers. Every warp stores its
//   partial sums; the last warp of a row group to finish adds them up, adds
//   scale * T B and writes the bf16 outputs, so no second pass over the partial sums runs.
// The GEMV is a programmatic dependent of the T kernel: it streams the weight at once and
// reads T and its counters only after griddepcontrol.wait.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdio>
#include <mutex>

#include "internal.h"
#include "nf4_device.cuh"

namespace qlora {
namespace {

constexpr int kDecThreads = 128;
// Weight rows per warp: one 16-row MMA group for M <= 8, two for M > 8 (the X fragments
// of 16 tokens are then shared by twice the rows); CTAs per SM follow the registers.
__host__ __device__ constexpr int rows_per_warp(bool tall) { return tall ? 32 : 16; }
__host__ __device__ constexpr int dec_ctas_per_sm(bool tall) { return tall ? 2 : 4; }
constexpr int kUnitK = 256;  // K covered by one warp step (4 lanes x 64)
constexpr int kTCtas = 8;    // cluster of the T kernel
constexpr int kTThreads = 256;

struct DecodeArgs {
  const uint8_t* codes;
  const uint8_t* c2;
  const float* c1;
  const float* mean;
  const uint16_t* X;
  const uint16_t* A;
  const uint16_t* B;
  int64_t M, N, K;
  int r;
  float scale;
  int splits, units_per, nunits;  // K is cut into `splits` ranges of `units_per` 256-units
  int row_groups;                 // groups of rows_per_warp(M > 8) rows of W
  float* part;      // [splits][row_groups][M][rows per warp] partial sums of X W_hat^T
  float* T;         // [M][r] T = X A
  float* T_save;    // optional copy of T for the backward pass
  int* counters;    // [row_groups] warps of the group that have stored their partials
  uint16_t* Y;      // [M][N]
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

__device__ __forceinline__ float bf16_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

__device__ __forceinline__ int64_t lmin(int64_t x, int64_t y) { return x < y ? x : y; }

// ---------------------------------------------------------------- T = X A
// Thread layout: 4 columns of A per thread (jq), k lanes (kl) striding over this CTA's
// share of K; X rows are read for all M tokens at once. Warp shuffles, then shared
// memory, then the cluster sum the partial products.
__global__ void __cluster_dims__(kTCtas, 1, 1) __launch_bounds__(kTThreads)
    k_decode_lora_down(const DecodeArgs a) {
  // the GEMV may start streaming the weight now; it waits for this grid before it
  // touches T or the counters
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ float wred[kTThreads / 32][16 * 64];
  __shared__ float cpart[16 * 64];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const int r = a.r;
  const int M = static_cast<int>(a.M);
  for (int i = static_cast<int>(rank) * kTThreads + tid; i < a.row_groups; i += kTCtas * kTThreads)
    a.counters[i] = 0;

  int jqn = 1;  // threads per A row: a power of two, 4 columns each
  while (jqn * 4 < r) jqn <<= 1;
  const int jq = tid & (jqn - 1), kl = tid / jqn, kls = kTThreads / jqn;
  const int j0 = jq * 4;
  const bool jlive = j0 < r;  // r is a multiple of 8, so j0 + 3 < r as well
  const int64_t kper = (a.K + 8 * kTCtas - 1) / (8 * kTCtas) * 8;  // K is a multiple of 64
  const int64_t k0 = static_cast<int64_t>(rank) * kper;
  const int64_t k1 = lmin(a.K, k0 + kper);
  float acc[16][4];
#pragma unroll
  for (int m = 0; m < 16; ++m)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[m][c] = 0.f;
  if (jlive) {
    // chunks of 8 consecutive k: every load of a chunk is issued before its math
    for (int64_t kc = k0 + 8 * kl; kc < k1; kc += 8 * kls) {
      float av[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(a.A + (kc + i) * r + j0));
        av[i][0] = bf16_to_f32(v.x & 0xFFFFu);
        av[i][1] = bf16_to_f32(v.x >> 16);
        av[i][2] = bf16_to_f32(v.y & 0xFFFFu);
        av[i][3] = bf16_to_f32(v.y >> 16);
      }
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        if (m < M) {
          const uint4 xv = __ldg(reinterpret_cast<const uint4*>(a.X + m * a.K + kc));
          const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float x = bf16_to_f32((i & 1) ? (xw[i >> 1] >> 16) : (xw[i >> 1] & 0xFFFFu));
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[m][c] = fmaf(x, av[i][c], acc[m][c]);
          }
        }
      }
    }
  }
  // lanes that share jq hold partial sums of the same outputs
  for (int o = jqn; o < 32; o <<= 1)
#pragma unroll
    for (int m = 0; m < 16; ++m)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[m][c] += __shfl_xor_sync(0xFFFFFFFFu, acc[m][c], o);
  if (lane < jqn && jlive)
#pragma unroll
    for (int m = 0; m < 16; ++m)
#pragma unroll
      for (int c = 0; c < 4; ++c) wred[warp][m * 64 + j0 + c] = acc[m][c];
  __syncthreads();
  const int mr = M * r;
  for (int e = tid; e < mr; e += kTThreads) {
    const int m = e / r, j = e % r;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kTThreads / 32; ++w) v += wred[w][m * 64 + j];
    cpart[e] = v;
  }
  cluster_sync_all();  // every CTA's partial sums are in its shared memory
  if (rank == 0) {
    for (int e = tid; e < mr; e += kTThreads) {
      float v = 0.f;
#pragma unroll
      for (int q = 0; q < kTCtas; ++q) v += ld_cluster_f32(&cpart[e], static_cast<uint32_t>(q));
      a.T[e] = v;
      if (a.T_save) a.T_save[e] = v;
    }
  }
  cluster_sync_all();  // no CTA leaves while rank 0 still reads its shared memory
}

// ---------------------------------------------------------------- X W_hat^T
// 64 consecutive bf16 of X row `row` starting at column k, as 32 packed pairs.
__device__ __forceinline__ void load_x64(const uint16_t* X, int64_t K, int64_t row, int64_t k,
                                         uint32_t (&x)[32]) {
  const uint4* p = reinterpret_cast<const uint4*>(X + row * K + k);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint4 v = __ldg(p + i);
    x[4 * i] = v.x;
    x[4 * i + 1] = v.y;
    x[4 * i + 2] = v.z;
    x[4 * i + 3] = v.w;
  }
}

// Fragment mapping of the weight tasks: mma.m16n8k16 with the dequantized weight as the
// A operand (16 weight rows) and X as the B operand (8 token columns). Lane (g = lane/4,
// t = lane%4) owns K columns kb .. kb + 63 (kb = unit * 256 + 64 t) of weight rows g
// and g + 8 of each 16-row group; MMA number j (0..15) of a unit takes from every lane
// the four columns kb + 4j .. kb + 4j + 3: A pairs (rows g and g + 8), B pairs (token
// g). Summation order over K does not matter, so this relabelling of the MMA's k index
// is free, and the unpacked pairs land directly in the A operand registers.

// Packed codes and block constants of one unit for this lane (rows beyond N are clamped
// and K beyond the matrix is clamped; their scale is forced to zero later).
template <int kGroups>
struct UnitCodes {
  uint4 q[kGroups][2][2];
  uint32_t e2[kGroups][2];
  float e1[kGroups][2];
};

// This lane's four weight rows (clamped to the last row; their scale is forced to zero
// later) as one base and 32-bit offsets from it, computed once per task.
template <int kGroups>
struct RowBases {
  const uint8_t* code;           // codes of the first row
  int64_t blk;                   // index of the first row's first 64-block
  int coff[kGroups][2];          // code byte offset of each row from `code`
  int boff[kGroups][2];          // block offset of each row from `blk`
};

template <int kGroups>
__device__ __forceinline__ void load_unit(const DecodeArgs& a, const RowBases<kGroups>& rb, int u,
                                          int t, int bpr, UnitCodes<kGroups>& c) {
  const int kbi = min(u * (kUnitK / 64) + t, bpr - 1);  // 64-block of this lane (clamped)
  const uint8_t* base = rb.code + kbi * 32;
  const int64_t jb = rb.blk + kbi;
#pragma unroll
  for (int q = 0; q < kGroups; ++q)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint8_t* p = base + rb.coff[q][h];
      c.q[q][h][0] = ldg_stream(p);
      c.q[q][h][1] = ldg_stream(p + 16);
      const int64_t j = jb + rb.boff[q][h];
      c.e2[q][h] = __ldg(a.c2 + j);
      c.e1[q][h] = __ldg(a.c1 + (j >> 8));
    }
}

template <bool kTall, int CB, int kGroups = kTall ? 2 : 1>
__device__ __forceinline__ void compute_unit(const DecodeArgs& a, int64_t rbase, int u, int g,
                                             int t, const UnitCodes<kGroups>& c, const float* t8,
                                             float mean, float (&acc)[kGroups][kTall ? 2 : 1][4]) {
  const int64_t K = a.K;
  const int64_t kraw = static_cast<int64_t>(u) * kUnitK + 64 * t;
  const bool kv = kraw < K;
  const int64_t kb = kv ? kraw : K - 64;
  // token rows this lane feeds to the B operand; tokens >= M compute columns nobody stores
  uint32_t xa[32], xb[32];
  load_x64(a.X, K, lmin(g, a.M - 1), kb, xa);
  if (kTall) load_x64(a.X, K, lmin(g + 8, a.M - 1), kb, xb);
#pragma unroll
  for (int q = 0; q < kGroups; ++q) {
    Nf4Lut lut[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const bool live = kv && (rbase + q * 16 + g + 8 * h) < a.N;
      build_lut<CB>(live ? block_scale_tab(t8, c.e2[q][h], c.e1[q][h], mean) : 0.f, lut[h]);
    }
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      uint32_t o0[4], o1[4];
      lut_decode8(w < 4 ? (&c.q[q][0][0].x)[w] : (&c.q[q][0][1].x)[w - 4], lut[0], o0);
      lut_decode8(w < 4 ? (&c.q[q][1][0].x)[w] : (&c.q[q][1][1].x)[w - 4], lut[1], o1);
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

template <bool kTall, int CB>
__device__ __forceinline__ void decode_weight_task(const DecodeArgs& a, int rg, int split,
                                                   int lane, const float* t8) {
  constexpr int kGroups = kTall ? 2 : 1;
  constexpr int kRowsPerWarp = rows_per_warp(kTall);
  const int g = lane >> 2, t = lane & 3;
  const int u0 = split * a.units_per;
  const int u1 = min(a.nunits, u0 + a.units_per);
  const float mean = *a.mean;
  const int64_t rbase = static_cast<int64_t>(rg) * kRowsPerWarp;
  float acc[kGroups][kTall ? 2 : 1][4];
#pragma unroll
  for (int q = 0; q < kGroups; ++q)
#pragma unroll
    for (int h = 0; h < (kTall ? 2 : 1); ++h)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[q][h][i] = 0.f;

  const int bpr = static_cast<int>(a.K / 64);
  RowBases<kGroups> rb;
  const int64_t row_g = lmin(rbase + g, a.N - 1);
  rb.code = a.codes + row_g * (a.K / 2);
  rb.blk = row_g * bpr;
#pragma unroll
  for (int q = 0; q < kGroups; ++q)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int dr = static_cast<int>(lmin(rbase + q * 16 + g + 8 * h, a.N - 1) - row_g);
      rb.coff[q][h] = dr * static_cast<int>(a.K / 2);
      rb.boff[q][h] = dr * bpr;
    }
  // two code buffers: the loads of unit u + 1 are in flight while unit u is expanded
  UnitCodes<kGroups> cb0, cb1;
  if (u0 < u1) load_unit(a, rb, u0, t, bpr, cb0);
  for (int u = u0; u < u1; u += 2) {
    if (u + 1 < u1) load_unit(a, rb, u + 1, t, bpr, cb1);
    compute_unit<kTall, CB>(a, rbase, u, g, t, cb0, t8, mean, acc);
    if (u + 1 < u1) {
      if (u + 2 < u1) load_unit(a, rb, u + 2, t, bpr, cb0);
      compute_unit<kTall, CB>(a, rbase, u + 1, g, t, cb1, t8, mean, acc);
    }
  }

  // C fragment: c0,c1 = (weight row g, tokens 2t, 2t+1), c2,c3 = (row g + 8, same tokens);
  // the second accumulator (M > 8) holds tokens 8 + 2t, 8 + 2t + 1.
  const int64_t M = a.M;
  float* pp = a.part + (static_cast<int64_t>(split) * a.row_groups + rg) * M * kRowsPerWarp;
#pragma unroll
  for (int q = 0; q < kGroups; ++q)
#pragma unroll
    for (int hm = 0; hm < (kTall ? 2 : 1); ++hm)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int rl = q * 16 + g + 8 * (i >> 1);
        const int m = 8 * hm + 2 * t + (i & 1);
        if (m < M) pp[m * kRowsPerWarp + rl] = acc[q][hm][i];
      }

  // T and the cleared counters come from the T kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __threadfence();
  __syncwarp();
  int last = 0;
  if (lane == 0) last = atomicAdd(a.counters + rg, 1) == a.splits - 1;
  last = __shfl_sync(0xFFFFFFFFu, last, 0);
  if (!last) return;
  __threadfence();  // the other warps' partial sums are visible from here on

  const int64_t row = rbase + lane;
  if (lane >= kRowsPerWarp || row >= a.N) return;
  float y[16], lora[16];
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    y[m] = 0.f;
    lora[m] = 0.f;
  }
  const int64_t sstride = static_cast<int64_t>(a.row_groups) * M * kRowsPerWarp;
  const float* p0 = a.part + static_cast<int64_t>(rg) * M * kRowsPerWarp + lane;
  for (int s = 0; s < a.splits; ++s) {
#pragma unroll
    for (int m = 0; m < 16; ++m)
      if (m < M) y[m] += __ldcg(p0 + s * sstride + m * kRowsPerWarp);
  }
  const int r = a.r;
  for (int j = 0; j < r; j += 4) {
    float bv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) bv[i] = bf16_to_f32(__ldg(a.B + (j + i) * a.N + row));
#pragma unroll
    for (int m = 0; m < 16; ++m)
      if (m < M) {
        const float4 tv = __ldcg(reinterpret_cast<const float4*>(a.T + m * r + j));
        lora[m] = fmaf(tv.x, bv[0], lora[m]);
        lora[m] = fmaf(tv.y, bv[1], lora[m]);
        lora[m] = fmaf(tv.z, bv[2], lora[m]);
        lora[m] = fmaf(tv.w, bv[3], lora[m]);
      }
  }
#pragma unroll
  for (int m = 0; m < 16; ++m)
    if (m < M) a.Y[m * a.N + row] = bf16_bits_rn(y[m] + a.scale * lora[m]);
}

// The two code buffers of the prefetch set the occupancy: 16 warps per SM with 16 rows per
// warp (M <= 8), 8 with 32 (M > 8), each without spills.
template <bool kTall, int CB>  // kTall: M > 8 (tokens 8..15 in the upper fragment rows); CB: codebook
__global__ void __launch_bounds__(kDecThreads, dec_ctas_per_sm(kTall)) k_decode_gemv(const DecodeArgs a) {
  __shared__ float t8[256];  // T8 by E4M3 code
  for (int i = threadIdx.x; i < 256; i += blockDim.x) t8[i] = t8_value(i);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int task = blockIdx.x * (kDecThreads / 32) + warp;
  if (task < a.row_groups * a.splits)
    decode_weight_task<kTall, CB>(a, task % a.row_groups, task / a.row_groups, lane, t8);
}

// ---------------------------------------------------------------- host side
struct DecodePlan {
  int splits, units_per, nunits, row_groups;
};

// K splits: enough warps for about two waves of the GEMV (16 or 8 resident warps per SM),
// but no more than K / (16 M): the partial sums (split x M x 4 bytes per row, written
// and read back through L2) stay at most half the code bytes.
DecodePlan plan_decode(const LinearShape& s) {
  DecodePlan p;
  p.nunits = static_cast<int>((s.K + kUnitK - 1) / kUnitK);
  const int rows = rows_per_warp(s.M > 8);
  p.row_groups = static_cast<int>((s.N + rows - 1) / rows);
  const int64_t per_sm = dec_ctas_per_sm(s.M > 8) * (kDecThreads / 32);
  const int64_t target = 2 * per_sm * num_sms();
  int64_t want = (target + p.row_groups - 1) / p.row_groups;
  want = std::min<int64_t>(want, std::max<int64_t>(1, s.K / (16 * std::max<int64_t>(1, s.M))));
  want = std::max<int64_t>(1, std::min<int64_t>(want, p.nunits));
  p.units_per = static_cast<int>((p.nunits + want - 1) / want);
  p.splits = (p.nunits + p.units_per - 1) / p.units_per;
  return p;
}

size_t part_bytes(const DecodePlan& p, const LinearShape& s) {
  return align_up(static_cast<size_t>(p.splits) * p.row_groups * s.M * rows_per_warp(s.M > 8) * 4,
                  256);
}
size_t t_bytes(const LinearShape& s) { return align_up(static_cast<size_t>(s.M) * s.r * 4, 256); }
size_t counter_bytes(const DecodePlan& p) { return align_up(static_cast<size_t>(p.row_groups) * 4, 256); }

// The T kernel, then the GEMV as its programmatic dependent.
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
  a.B = B;
  a.M = s.M;
  a.N = s.N;
  a.K = s.K;
  a.r = s.r;
  a.scale = s.scale;
  a.splits = p.splits;
  a.units_per = p.units_per;
  a.nunits = p.nunits;
  a.row_groups = p.row_groups;
  a.part = reinterpret_cast<float*>(scratch);
  a.T = reinterpret_cast<float*>(scratch + part_bytes(p, s));
  a.counters = reinterpret_cast<int*>(scratch + part_bytes(p, s) + t_bytes(s));
  a.T_save = T_save;
  a.Y = Y;
  note_launches(2);  // this kernel and the GEMV below
  k_decode_lora_down<<<kTCtas, kTThreads, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e);
  const int64_t warps = static_cast<int64_t>(p.row_groups) * p.splits;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((warps + kDecThreads / 32 - 1) / (kDecThreads / 32)));
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (w.codebook == 1)
    e = s.M > 8 ? cudaLaunchKernelEx(&cfg, k_decode_gemv<true, 1>, a)
                : cudaLaunchKernelEx(&cfg, k_decode_gemv<false, 1>, a);
  else
    e = s.M > 8 ? cudaLaunchKernelEx(&cfg, k_decode_gemv<true, 0>, a)
                : cudaLaunchKernelEx(&cfg, k_decode_gemv<false, 0>, a);
  if (e != cudaSuccess) return cuda_status(e);
  return QLORA_OK;
}

size_t decode_scratch_bytes(const DecodePlan& p, const LinearShape& s) {
  return part_bytes(p, s) + t_bytes(s) + counter_bytes(p);
}

}  // namespace

size_t decode_workspace(const LinearShape& s) {
  return decode_scratch_bytes(plan_decode(s), s) + 256;
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
  if (w.codebook < 0 || w.codebook >= kCodebooks) return QLORA_ERR_INVALID_ARG;
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
  const size_t per_split = static_cast<size_t>(p.row_groups) * M * rows_per_warp(M > 8) * 4;
  const size_t fixed = t_bytes(s) + counter_bytes(p) + 512;
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
  // Every partial sum is written by the GEMV before it is read, and the T kernel clears
  // the arrival counters, so nothing left in the array by an earlier call matters.
  return launch_decode(X, w, A, B, s, p, Y, T_save, static_cast<char*>(scratch),
                       static_cast<cudaStream_t>(stream));
}

