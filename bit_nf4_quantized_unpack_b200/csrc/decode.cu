// decode.cu -- the QLoRA linear forward for M <= 16 tokens (decode), which is bound by
// reading the packed weight (0.516 B per parameter) and by the work of expanding it.
//
//   Y = bf16(X W_hat^T + scale (X A) B)    (page "QLoRA", itwiki.kr, section "계산 방식";
//                                           alpha/r from page "quantization", minnong511)
//
// Two launches per call:
// k_decode_prep: zeroes T and the arrival counters of the call. It is a programmatic
//   dependent of whatever ran before on the stream (it launches while that kernel drains
//   and waits for it to complete before it writes), and it lets the main kernel launch at
//   once.
// k_decode_gemv (its programmatic dependent): one CTA of 16 warps per SM. CTA c owns one
//   K split (split c % splits) and the row groups c / splits, + cps, ... of it. It builds
//   its constant tables, waits for k_decode_prep, stages the split's columns of X in
//   shared memory once (padded so that the MMA operand loads are conflict-free), then
//   * its 15 weight warps each take one group of 16 weight rows over the split: lanes
//     stream 32 bytes of packed codes per row with 128-bit loads (the next 256-wide unit
//     while the current one is expanded), double-dequantize them straight into the A
//     fragments of mma.m16n8k16 (X is the B operand; the dequantized weight never leaves
//     registers) and store the split's partial sums; the last warp of a row group to
//     arrive adds the splits up in a fixed order, adds scale * T B and writes bf16 Y;
//   * its last warp computes T = X A over its share of the split's rows from the staged X
//     and adds it into T with fp32 reductions (so T's summation order varies from run to
//     run, within fp32 rounding; Y's does not); the finishers wait, bounded, until every
//     share is in.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdio>
#include <mutex>

#include "internal.h"
#include "nf4_device.cuh"

namespace qlora {
namespace {

// Weight rows per warp task: one 16-row MMA group (for M > 8 the warp issues a second MMA
// per step for tokens 8..15 with the same A fragments).
constexpr int kRowsPerWarp = 16;
// One CTA per SM: 16 warps at <= 128 registers; the last warp of a CTA computes its share
// of T, the others take weight rows.
constexpr int kDecThreads = 512;
constexpr int kWeightWarps = kDecThreads / 32 - 1;
constexpr int kUnitK = 256;  // K covered by one warp step (4 lanes x 64)

// X stage: each 64-column block of a token's row takes 128 bytes at a 144-byte stride,
// and token rows are xs_tok bytes apart with xs_tok = 64 (mod 128). A B-fragment load
// (lane (g, t) reads 16 bytes of block t of token g) then spreads over all eight 16-byte
// bank groups.
constexpr int kXBlkStride = 144;
constexpr int kXStageMax = 80 * 1024;
constexpr uint32_t kPairTabBytes = 65536;
// A T share stages up to kTChunkRows rows of A at a time.
constexpr int kTChunkRows = 64;
constexpr int kPrefetchRank = 16;  // ranks of B a finisher fetches before it knows it is one
__host__ __device__ constexpr int a_chunk_bytes(int r) { return kTChunkRows * r * 2; }
// the finishers stage T (M x r fp32) in the same area
static_assert(4 * kDecodeMaxM <= 2 * kTChunkRows, "T fits the A-chunk area");
// Dynamic shared memory: the 64 KB pair table at a 64 KB-aligned address (up to 64 KB of
// alignment slack below it), the X stage, T8 (1 KB) and the A chunk; the last three are
// placed in the slack when they fit there, else above the table.
__host__ __device__ constexpr uint32_t dec_smem_bytes(int xs_bytes, int r) {
  return 2 * kPairTabBytes + static_cast<uint32_t>(xs_bytes) + 1024u +
         static_cast<uint32_t>(a_chunk_bytes(r));
}
constexpr uint32_t kDecSmemMax = dec_smem_bytes(kXStageMax, 64);

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
  int row_groups;                 // groups of kRowsPerWarp rows of W
  int cps;                        // CTAs per split (grid = splits x cps)
  int xs_tok;                     // bytes between token rows of the X stage
  int xs_bytes;                   // bytes of the X stage (M x xs_tok)
  float* part;      // [splits][row_groups][M][kRowsPerWarp] partial sums of X W_hat^T
  float* T;         // [M][r] T = X A (zeroed by k_decode_prep)
  float* T_save;    // optional copy of T for the backward pass
  int* counters;    // [row_groups] warps of the group that have stored their partials
  int* t_count;     // T shares added so far
  int* err;         // device error word
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

__device__ __forceinline__ float bf16_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

__device__ __forceinline__ int64_t lmin(int64_t x, int64_t y) { return x < y ? x : y; }

__device__ __forceinline__ uint64_t lds_b64(uint32_t addr) {
  uint64_t v;
  asm volatile("ld.shared.b64 %0, [%1];" : "=l"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint4 lds_b128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts_b128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ uint2 lds_b64x2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}
__device__ __forceinline__ int atom_add_acq_rel_gpu(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// ---------------------------------------------------------------- call set-up
__global__ void __launch_bounds__(256) k_decode_prep(float* T, int mr, int* counters, int nc,
                                                     int* t_count) {
  // the main kernel may launch now (it waits for this grid before it reads its inputs);
  // this grid waits for the kernel before it (which may still read T or the counters of
  // the previous call) before it writes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int stride = gridDim.x * blockDim.x;
  const int i0 = blockIdx.x * blockDim.x + threadIdx.x;
  for (int i = i0; i < mr; i += stride) T[i] = 0.f;
  for (int i = i0; i < nc; i += stride) counters[i] = 0;
  if (i0 == 0) *t_count = 0;
}

// ---------------------------------------------------------------- X W_hat^T
// Fragment mapping of the weight tasks: mma.m16n8k16 with the dequantized weight as the
// A operand (16 weight rows) and X as the B operand (8 token columns). Lane (g = lane/4,
// t = lane%4) owns K columns kb .. kb + 63 (kb = unit * 256 + 64 t) of weight rows g
// and g + 8 of each 16-row group; MMA number j (0..15) of a unit takes from every lane
// the four columns kb + 4j .. kb + 4j + 3: A pairs (rows g and g + 8), B pairs (token
// g). Summation order over K does not matter, so this relabelling of the MMA's k index
// is free, and the expanded pairs land directly in the A operand registers.
//
// Two ways to expand a 64-block of codes, both giving bf16_rn(fl32(L[code] * s)) bit for
// bit; a warp uses both so that neither the integer ALU nor the shared-memory pipe
// alone bounds it (three quarters pair table for M <= 8, half for M > 8):
//  * the pair table: every byte of codes (two weights) is the index of a shared-memory
//    entry holding the two fp32 levels; one packed fp32 multiply by s and one bf16x2
//    conversion give the operand pair. Per byte: one byte permute to form the address,
//    one 8-byte shared load, one f32x2 multiply, one conversion.
//  * the permute table (build_lut / lut_decode8 in nf4_device.cuh): a per-block
//    16-entry bf16 table in registers, indexed by the codes through byte permutes.

// Byte-pair level table: entry e (the code byte e: code e & 15 in its low nibble, e >> 4
// in its high nibble) holds (L[e & 15], L[e >> 4]) as two fp32. Copy c (c = lane % 16)
// of entry e lives at byte e * 256 + c * 8 of a 64 KB-aligned region, so the 16 lanes of
// a half-warp read 16 distinct bank pairs whatever their bytes; the uniform codebook's
// copies take bytes 128..255 of each 256-byte row. With the region 64 KB-aligned, one
// byte permute builds the shared address from the code byte and a per-lane constant.

// Eight codes (one word of packed codes) -> four bf16x2 operand registers through the
// pair table (o[i] = elements 2i, 2i + 1); `lane_bits` holds the lane's copy offset in
// byte 0 and byte 2 of the table's base in byte 2; s2 is the block scale in both halves.
__device__ __forceinline__ void pair_decode8(uint32_t w, uint32_t lane_bits, uint64_t s2,
                                             uint32_t (&o)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t addr = prmt(w, lane_bits, 0x7604u | (static_cast<uint32_t>(i) << 4));
    float lo, hi;
    f2_unpack(f2_mul(lds_b64(addr), s2), lo, hi);
    o[i] = pack_bf16x2_rn(lo, hi);
  }
}

// Packed codes and block constants of one unit for this lane (rows beyond N are clamped
// and K beyond the matrix is clamped; their scale is forced to zero later).
struct UnitCodes {
  uint4 q[2][2];  // [row g / g + 8][first / second 16 bytes]
  uint32_t e2[2];
  float e1[2];
};

// This lane's weight rows (clamped to the last row; their scale is forced to zero later)
// as one base and 32-bit offsets from it, computed once per task.
struct RowBases {
  const uint8_t* code;  // codes of row g
  int64_t blk;          // index of row g's first 64-block
  int coff;             // code byte offset of row g + 8 from `code`
  int boff;             // block offset of row g + 8 from `blk`
};

// Streamed 16-byte load of packed codes that also asks L2 to fetch the whole 256-byte
// segment (the next unit of the same row).
__device__ __forceinline__ uint4 ldg_codes(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void load_unit(const DecodeArgs& a, const RowBases& rb, int u, int t,
                                          int bpr, UnitCodes& c) {
  const int kbi = min(u * (kUnitK / 64) + t, bpr - 1);  // 64-block of this lane (clamped)
  const uint8_t* base = rb.code + kbi * 32;
  const int64_t jb = rb.blk + kbi;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint8_t* p = base + (h ? rb.coff : 0);
    c.q[h][0] = ldg_codes(p);
    c.q[h][1] = ldg_codes(p + 16);
    const int64_t j = jb + (h ? rb.boff : 0);
    c.e2[h] = __ldg(a.c2 + j);
    c.e1[h] = __ldg(a.c1 + (j >> 8));
  }
}

// One unit: the codes of row g go through the pair table, those of row g + 8 through the
// permute table, or through the pair table as well when kAllPair. xs0 / xs1: this lane's
// tokens' rows of the X stage (tokens g and, for M > 8, g + 8).
template <bool kTall, int CB, bool kAllPair>
__device__ __forceinline__ void compute_unit(const DecodeArgs& a, int64_t rbase, int u, int u0,
                                             int nblk, int g, int t, const UnitCodes& c,
                                             const float* t8, float mean, uint32_t lane_bits,
                                             uint32_t xs0, uint32_t xs1,
                                             float (&acc)[kTall ? 2 : 1][4]) {
  const int blk = (u - u0) * (kUnitK / 64) + t;  // block of the split
  const bool kv = blk < nblk;                    // false past the end of K
  const uint32_t xoff = static_cast<uint32_t>(min(blk, nblk - 1) * kXBlkStride);
  const bool live0 = kv && (rbase + g) < a.N, live1 = kv && (rbase + g + 8) < a.N;
  const float s0 = live0 ? block_scale_tab(t8, c.e2[0], c.e1[0], mean) : 0.f;
  const float s1 = live1 ? block_scale_tab(t8, c.e2[1], c.e1[1], mean) : 0.f;
  const uint64_t s2 = f2_pack(s0, s0);
  const uint64_t s2b = f2_pack(s1, s1);
  Nf4Lut lut;
  if (!kAllPair) build_lut<CB>(s1, lut);
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    // this word's 8 columns of X for the lane's token(s), just before their MMAs
    const uint4 xa = lds_b128(xs0 + xoff + 16 * w);
    uint32_t o0[4], o1[4];
    pair_decode8(w < 4 ? (&c.q[0][0].x)[w] : (&c.q[0][1].x)[w - 4], lane_bits, s2, o0);
    if (kAllPair)
      pair_decode8(w < 4 ? (&c.q[1][0].x)[w] : (&c.q[1][1].x)[w - 4], lane_bits, s2b, o1);
    else
      lut_decode8(w < 4 ? (&c.q[1][0].x)[w] : (&c.q[1][1].x)[w - 4], lut, o1);
    mma_bf16_16816(acc[0], o0[0], o1[0], o0[1], o1[1], xa.x, xa.y);
    mma_bf16_16816(acc[0], o0[2], o1[2], o0[3], o1[3], xa.z, xa.w);
    if (kTall) {
      const uint4 xb = lds_b128(xs1 + xoff + 16 * w);
      mma_bf16_16816(acc[kTall ? 1 : 0], o0[0], o1[0], o0[1], o1[1], xb.x, xb.y);
      mma_bf16_16816(acc[kTall ? 1 : 0], o0[2], o1[2], o0[3], o1[3], xb.z, xb.w);
    }
  }
}

// Bounded wait of a finisher for every T share of the call (lane 0 spins; false on
// timeout, after recording it).
__device__ __forceinline__ bool wait_t_complete(const DecodeArgs& a, int lane) {
  int ok = 1;
  if (lane == 0) {
    const int need = a.splits * a.cps;
    if (ld_acquire_gpu(a.t_count) < need) {
      const uint64_t t0 = global_timer_ns();
      for (uint32_t it = 0;; ++it) {
        if (ld_acquire_gpu(a.t_count) >= need) break;
        if ((it & 63) == 63 && global_timer_ns() - t0 > kWaitTimeoutNs) {
          atomicCAS(a.err, 0, kErrTimeoutDecode);
          ok = 0;
          break;
        }
      }
    }
  }
  return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

template <bool kTall, int CB>
__device__ __forceinline__ void decode_weight_task(const DecodeArgs& a, int rg, int split,
                                                   int nblk, int lane, const float* t8,
                                                   uint32_t lane_bits, uint32_t xs,
                                                   uint32_t ts) {
  const int g = lane >> 2, t = lane & 3;
  const int u0 = split * a.units_per;
  const int u1 = min(a.nunits, u0 + a.units_per);
  const float mean = *a.mean;
  const int64_t rbase = static_cast<int64_t>(rg) * kRowsPerWarp;
  const uint32_t xs0 = xs + static_cast<uint32_t>(min(g, static_cast<int>(a.M) - 1) * a.xs_tok);
  const uint32_t xs1 =
      xs + static_cast<uint32_t>(min(g + 8, static_cast<int>(a.M) - 1) * a.xs_tok);
  float acc[kTall ? 2 : 1][4];
#pragma unroll
  for (int h = 0; h < (kTall ? 2 : 1); ++h)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[h][i] = 0.f;

  const int bpr = static_cast<int>(a.K / 64);
  RowBases rb;
  const int64_t row_g = lmin(rbase + g, a.N - 1);
  rb.code = a.codes + row_g * (a.K / 2);
  rb.blk = row_g * bpr;
  const int dr = static_cast<int>(lmin(rbase + g + 8, a.N - 1) - row_g);
  rb.coff = dr * static_cast<int>(a.K / 2);
  rb.boff = dr * bpr;
  // two code buffers: the loads of unit u + 1 are in flight while unit u is expanded.
  // Which table each row takes: M <= 8, row g + 8 of odd units through the pair table too
  // (three quarters pair table); M > 8, half and half (its second X fragment loads take
  // shared-memory bandwidth of their own).
  UnitCodes cb0, cb1;
  if (u0 < u1) load_unit(a, rb, u0, t, bpr, cb0);
  for (int u = u0; u < u1; u += 2) {
    if (u + 1 < u1) load_unit(a, rb, u + 1, t, bpr, cb1);
    compute_unit<kTall, CB, false>(a, rbase, u, u0, nblk, g, t, cb0, t8, mean, lane_bits, xs0,
                                   xs1, acc);
    if (u + 1 < u1) {
      if (u + 2 < u1) load_unit(a, rb, u + 2, t, bpr, cb0);
      compute_unit<kTall, CB, !kTall>(a, rbase, u + 1, u0, nblk, g, t, cb1, t8, mean, lane_bits,
                                      xs0, xs1, acc);
    }
  }

  // C fragment: c0,c1 = (weight row g, tokens 2t, 2t+1), c2,c3 = (row g + 8, same tokens);
  // the second accumulator (M > 8) holds tokens 8 + 2t, 8 + 2t + 1.
  const int64_t M = a.M;
  float* pp = a.part + (static_cast<int64_t>(split) * a.row_groups + rg) * M * kRowsPerWarp;
#pragma unroll
  for (int hm = 0; hm < (kTall ? 2 : 1); ++hm)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int rl = g + 8 * (i >> 1);
      const int m = 8 * hm + 2 * t + (i & 1);
      if (m < M) pp[m * kRowsPerWarp + rl] = acc[hm][i];
    }

  // The finisher's operands that are ready now: B[j][row] for the first kPrefetchRank j of
  // this lane's row (lane (rl, half) = (lane % 16, lane / 16)), as bf16 pairs; in flight
  // while the arrival is counted.
  const int rl = lane & 15, half = lane >> 4;
  const int64_t row = rbase + rl;
  const int64_t rowc = lmin(row, a.N - 1);
  const int r = a.r;
  uint32_t bq[kPrefetchRank / 2];
#pragma unroll
  for (int i = 0; i < kPrefetchRank / 2; ++i)
    if (2 * i < r)
      bq[i] = static_cast<uint32_t>(__ldg(a.B + (2 * i) * a.N + rowc)) |
              (static_cast<uint32_t>(__ldg(a.B + (2 * i + 1) * a.N + rowc)) << 16);

  // Arrival: the warp's partial sums are ordered before the count (release), and the
  // last warp of the row group sees every other warp's (acquire). The counters come
  // zeroed from k_decode_prep.
  __syncwarp();
  int last = 0;
  if (lane == 0) last = atom_add_acq_rel_gpu(a.counters + rg, 1) == a.splits - 1;
  last = __shfl_sync(0xFFFFFFFFu, last, 0);
  if (!last) return;
  if (!wait_t_complete(a, lane)) return;
  __syncwarp();

  // T (complete now) into the CTA's A-chunk area of shared memory, by asynchronous copies
  // in flight with the partial-sum loads below. This CTA's T warp has stopped using the
  // area (it counted its share in after its last chunk), and every finisher of the CTA
  // writes the same values there.
  const int mr = static_cast<int>(M) * r;  // a multiple of 8
  for (int e = 4 * lane; e < mr; e += 128) cp_async16(ts + 4 * e, a.T + e);
  asm volatile("cp.async.commit_group;" ::: "memory");

  // the splits' partial sums of tokens m = half, half + 2, ..., added four splits at a
  // time in a fixed order
  float y[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) y[i] = 0.f;
  const int64_t sstride = static_cast<int64_t>(a.row_groups) * M * kRowsPerWarp;
  const float* p0 = a.part + static_cast<int64_t>(rg) * M * kRowsPerWarp + rl;
  int s = 0;
  for (; s + 4 <= a.splits; s += 4) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int m = 2 * i + half;
      if (m < M) {
        const float* q = p0 + s * sstride + m * kRowsPerWarp;
        const float v0 = __ldcg(q), v1 = __ldcg(q + sstride);
        const float v2 = __ldcg(q + 2 * sstride), v3 = __ldcg(q + 3 * sstride);
        y[i] += (v0 + v1) + (v2 + v3);
      }
    }
  }
  for (; s < a.splits; ++s) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int m = 2 * i + half;
      if (m < M) y[i] += __ldcg(p0 + s * sstride + m * kRowsPerWarp);
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncwarp();

  if (row >= a.N) return;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = 2 * i + half;
    if (m < M) {
      float lora = 0.f;
#pragma unroll
      for (int j4 = 0; j4 < kPrefetchRank / 4; ++j4)
        if (4 * j4 < r) {
          const uint4 tv = lds_b128(ts + static_cast<uint32_t>((m * r + 4 * j4) * 4));
          const uint32_t b01 = bq[2 * j4], b23 = bq[2 * j4 + 1];
          lora = fmaf(__uint_as_float(tv.x), bf16_to_f32(b01 & 0xFFFFu), lora);
          lora = fmaf(__uint_as_float(tv.y), bf16_to_f32(b01 >> 16), lora);
          lora = fmaf(__uint_as_float(tv.z), bf16_to_f32(b23 & 0xFFFFu), lora);
          lora = fmaf(__uint_as_float(tv.w), bf16_to_f32(b23 >> 16), lora);
        }
      for (int j = kPrefetchRank; j < r; j += 4) {  // ranks above kPrefetchRank
        const uint4 tv = lds_b128(ts + static_cast<uint32_t>((m * r + j) * 4));
        lora = fmaf(__uint_as_float(tv.x), bf16_to_f32(__ldg(a.B + j * a.N + rowc)), lora);
        lora = fmaf(__uint_as_float(tv.y), bf16_to_f32(__ldg(a.B + (j + 1) * a.N + rowc)), lora);
        lora = fmaf(__uint_as_float(tv.z), bf16_to_f32(__ldg(a.B + (j + 2) * a.N + rowc)), lora);
        lora = fmaf(__uint_as_float(tv.w), bf16_to_f32(__ldg(a.B + (j + 3) * a.N + rowc)), lora);
      }
      a.Y[m * a.N + row] = bf16_bits_rn(y[i] + a.scale * lora);
    }
  }
}

// ---------------------------------------------------------------- T = X A
// The CTA's share of T: rows [k0, k1) of A (inside its split, so X comes from the stage).
// Rows of A are staged kTChunkRows at a time with asynchronous 16-byte copies (one
// latency round per chunk). Lane (jq, kq): columns 4 jq .. 4 jq + 3 of A, row octets kq,
// kq + kqn, ... of the chunk, every token; the kqn lanes of a column group then add
// their sums with shuffles and lane kq = 0 adds them into T.
__device__ __forceinline__ void decode_t_share(const uint16_t* __restrict__ A, float* T,
                                               float* T_save, int* t_count, int shares, int r,
                                               int M, int xs_tok, int64_t kbeg, int64_t k0,
                                               int64_t k1, int lane, uint32_t xs, uint32_t as) {
  int jqn = 2;  // lanes per row: a power of two with 4 jqn >= r
  while (jqn * 4 < r) jqn <<= 1;
  const int kqn = 32 / jqn;  // lanes along the rows (>= 2)
  const int jq = lane & (jqn - 1), kq = lane / jqn;
  const int j0 = jq * 4;
  const bool jlive = j0 < r;  // r is a multiple of 8, so j0 + 3 < r as well
  float acc[16][4];
#pragma unroll
  for (int m = 0; m < 16; ++m)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[m][c] = 0.f;
  for (int64_t kc = k0; kc < k1; kc += kTChunkRows) {  // k0, k1 are multiples of 8
    const int rows = static_cast<int>(lmin(kTChunkRows, k1 - kc));
    const int pieces = rows * r / 8;  // 16-byte pieces of the chunk
    for (int i = lane; i < pieces; i += 32) cp_async16(as + 16 * i, A + kc * r + 8 * i);
    cp_async_wait_all();
    __syncwarp();
    if (jlive) {
      for (int o = kq; o < rows / 8; o += kqn) {
        float av[8][4];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint2 v = lds_b64x2(as + static_cast<uint32_t>(((8 * o + e) * r + j0) * 2));
          av[e][0] = bf16_to_f32(v.x & 0xFFFFu);
          av[e][1] = bf16_to_f32(v.x >> 16);
          av[e][2] = bf16_to_f32(v.y & 0xFFFFu);
          av[e][3] = bf16_to_f32(v.y >> 16);
        }
        const int64_t kk = kc + 8 * o - kbeg;
        const uint32_t xo = static_cast<uint32_t>((kk >> 6) * kXBlkStride + (kk & 63) * 2);
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          if (m < M) {
            const uint4 xv = lds_b128(xs + static_cast<uint32_t>(m * xs_tok) + xo);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const uint32_t xw = (e >> 1) == 0 ? xv.x : (e >> 1) == 1 ? xv.y : (e >> 1) == 2 ? xv.z : xv.w;
              const float x = bf16_to_f32((e & 1) ? (xw >> 16) : (xw & 0xFFFFu));
#pragma unroll
              for (int c = 0; c < 4; ++c) acc[m][c] = fmaf(x, av[e][c], acc[m][c]);
            }
          }
        }
      }
    }
    __syncwarp();  // the chunk is read before the next one overwrites it
  }
  for (int off = jqn; off < 32; off <<= 1)
#pragma unroll
    for (int m = 0; m < 16; ++m)
      if (m < M)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[m][c] += __shfl_xor_sync(0xFFFFFFFFu, acc[m][c], off);
  // T was zeroed by k_decode_prep; one 4-wide reduction per token and column quad (all
  // CTAs add into the same M x r floats, so fewer, wider operations queue less at L2)
  if (jlive && kq == 0 && k0 < k1) {
#pragma unroll
    for (int m = 0; m < 16; ++m)
      if (m < M) red_add_v4(T + m * r + j0, acc[m][0], acc[m][1], acc[m][2], acc[m][3]);
  }
  // the share is counted after its additions (release); the last share's warp sees all
  // of T (acquire) and copies it out
  __syncwarp();
  int last = 0;
  if (lane == 0) last = atom_add_acq_rel_gpu(t_count, 1) == shares - 1;
  last = __shfl_sync(0xFFFFFFFFu, last, 0);
  if (last && T_save) {
    __syncwarp();
    for (int e = lane; e < M * r; e += 32) T_save[e] = __ldcg(T + e);
  }
}

// ---------------------------------------------------------------- the main kernel
template <bool kTall, int CB>  // kTall: M > 8 (tokens 8..15 in the upper fragment rows); CB: codebook
__global__ void __launch_bounds__(kDecThreads, 1) k_decode_gemv(const DecodeArgs a) {
  extern __shared__ __align__(16) uint8_t dsm[];
  const uint32_t sbase = smem_u32(dsm);
  const uint32_t tab = (sbase + kPairTabBytes - 1) & ~(kPairTabBytes - 1);
  // the X stage, T8 and the A chunk go below the table while they fit there, else above
  uint32_t lo_used = 0, hi_used = (tab - sbase) + kPairTabBytes;
  auto place = [&](uint32_t bytes) {
    if (lo_used + bytes <= tab - sbase) {
      lo_used += bytes;
      return lo_used - bytes;
    }
    hi_used += bytes;
    return hi_used - bytes;
  };
  const uint32_t xs_off = place(static_cast<uint32_t>(a.xs_bytes));
  const uint32_t t8_off = place(1024u);
  const uint32_t as_off = place(static_cast<uint32_t>(a_chunk_bytes(a.r)));
  const uint32_t xs = sbase + xs_off;
  float* t8 = reinterpret_cast<float*>(dsm + t8_off);
  uint8_t* tabp = dsm + (tab - sbase);
  const int split = blockIdx.x % a.splits, cidx = blockIdx.x / a.splits;
  const int u0 = split * a.units_per;
  const int u1 = min(a.nunits, u0 + a.units_per);
  const int64_t kbeg = static_cast<int64_t>(u0) * kUnitK;
  const int64_t kend = lmin(a.K, static_cast<int64_t>(u1) * kUnitK);
  const int nblk = static_cast<int>((kend - kbeg) / 64);  // K is a multiple of 64
  const int M = static_cast<int>(a.M);

  // the next kernel on the stream may launch now (a programmatic dependent waits for this
  // grid to complete before it reads what it writes)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // the constant tables: T8 and the pair table, 256 entries x 16 copies; thread i writes
  // entry i / 16, copy i % 16 (its low level index (i / 16) % 16 is the same at every step)
  for (int i = threadIdx.x; i < 256; i += blockDim.x) t8[i] = t8_value(i);
  {
    const float lo = code_level_rt<CB>((threadIdx.x >> 4) & 15);
    for (int i = threadIdx.x; i < 256 * 16; i += blockDim.x) {
      const int e = i >> 4, cp = i & 15;
      *reinterpret_cast<float2*>(tabp + e * 256 + CB * 128 + cp * 8) =
          make_float2(lo, code_level_rt<CB>(e >> 4));
    }
  }
  // k_decode_prep, and so every kernel before it on the stream, is complete from here on:
  // X, A and the cleared T and counters are ready
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // X columns [kbeg, kend) of every token, 16 bytes per thread and step: the loads of
  // four steps are issued before their stores
  {
    const int n16 = M * nblk * 8;
    for (int i0 = threadIdx.x; i0 < n16; i0 += 4 * blockDim.x) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * blockDim.x;
        if (i < n16) {
          const int m = i / (nblk * 8), rem = i - m * (nblk * 8);
          v[u] = __ldg(reinterpret_cast<const uint4*>(a.X + m * a.K + kbeg + rem * 8));
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * blockDim.x;
        if (i < n16) {
          const int m = i / (nblk * 8), rem = i - m * (nblk * 8);
          sts_b128(xs + static_cast<uint32_t>(m * a.xs_tok + (rem >> 3) * kXBlkStride +
                                               (rem & 7) * 16),
                   v[u]);
        }
      }
    }
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kW = kWeightWarps;
  if (warp == kW) {
    // this CTA's share of the split's rows of A
    const int64_t share = ((kend - kbeg + a.cps - 1) / a.cps + 7) / 8 * 8;
    const int64_t k0 = lmin(kend, kbeg + cidx * share);
    const int64_t k1 = lmin(kend, k0 + share);
    decode_t_share(a.A, a.T, a.T_save, a.t_count, a.splits * a.cps, a.r, M, a.xs_tok, kbeg, k0,
                   k1, lane, xs, sbase + as_off);
    return;
  }
  const uint32_t lane_bits =
      static_cast<uint32_t>((lane & 15) * 8 + CB * 128) | (tab & 0x00FF0000u);
  for (int rg = cidx + a.cps * warp; rg < a.row_groups; rg += a.cps * kW)
    decode_weight_task<kTall, CB>(a, rg, split, nblk, lane, t8, lane_bits, xs, sbase + as_off);
}

// ---------------------------------------------------------------- host side
struct DecodePlan {
  int splits, units_per, nunits, row_groups, cps, xs_tok;
};

int x_stage_tok(int units_per) {
  const int raw = units_per * (kUnitK / 64) * kXBlkStride;
  return (raw + 63) / 128 * 128 + 64;  // >= raw, = 64 (mod 128)
}

size_t part_bytes(const DecodePlan& p, const LinearShape& s) {
  return align_up(static_cast<size_t>(p.splits) * p.row_groups * s.M * kRowsPerWarp * 4, 256);
}
size_t t_bytes(const LinearShape& s) { return align_up(static_cast<size_t>(s.M) * s.r * 4, 256); }
size_t counter_bytes(const DecodePlan& p) {
  return align_up(static_cast<size_t>(p.row_groups) * 4 + 4, 256);  // + the T count
}
size_t decode_scratch_bytes(const DecodePlan& p, const LinearShape& s) {
  return part_bytes(p, s) + t_bytes(s) + counter_bytes(p);
}

// K splits and CTAs per split. CTA c takes split c % splits and row groups c / splits,
// + cps, ...; each of its weight warps one row group at a time over the whole split. The
// choice minimises the units of the busiest warp (each task charged one extra unit for
// its pipeline fill and its partial-sum store, and a CTA with fewer than three quarters
// of its weight warps busy charged for the bandwidth it leaves unused), subject to the X
// stage fitting its shared-memory budget, at most K / (16 M) splits (the partial sums,
// split x M x 4 bytes per row, stay at most half the code bytes) and the scratch fitting
// `max_scratch`. Ties go to fewer splits. Returns splits = 0 when nothing fits.
DecodePlan plan_decode(const LinearShape& s, size_t max_scratch = ~size_t{0}) {
  DecodePlan p;
  p.nunits = static_cast<int>((s.K + kUnitK - 1) / kUnitK);
  p.row_groups = static_cast<int>((s.N + kRowsPerWarp - 1) / kRowsPerWarp);
  const int64_t W = kWeightWarps;
  const int64_t sms = num_sms();
  const int64_t max_splits =
      std::max<int64_t>(1, std::min<int64_t>(p.nunits, s.K / (16 * std::max<int64_t>(1, s.M))));
  double best_cost = -1.0;
  p.splits = 0;
  p.units_per = p.nunits;
  p.cps = 1;
  p.xs_tok = x_stage_tok(p.nunits);
  for (int up = p.nunits; up >= 1; --up) {
    const int64_t splits = (p.nunits + up - 1) / up;
    if (splits > max_splits || splits > sms) continue;
    if (s.M * x_stage_tok(up) > kXStageMax) continue;
    DecodePlan c = p;
    c.splits = static_cast<int>(splits);
    c.units_per = up;
    if (decode_scratch_bytes(c, s) > max_scratch) continue;
    const int64_t cps = std::max<int64_t>(1, std::min<int64_t>(sms / splits, p.row_groups));
    const int64_t per_cta = (p.row_groups + cps - 1) / cps;
    const int64_t tasks = (per_cta + W - 1) / W;
    const int64_t busy = std::min<int64_t>(per_cta, W);
    const double want = 0.75 * static_cast<double>(W);
    const double cost = static_cast<double>(tasks * (up + 1)) *
                        (static_cast<double>(busy) < want ? want / static_cast<double>(busy) : 1.0);
    if (best_cost < 0.0 || cost < best_cost) {
      best_cost = cost;
      p.splits = static_cast<int>(splits);
      p.units_per = up;
      p.cps = static_cast<int>(cps);
    }
  }
  p.xs_tok = x_stage_tok(p.units_per);
  return p;
}

template <bool kTall, int CB>
cudaError_t launch_gemv(cudaLaunchConfig_t& cfg, const DecodeArgs& a) {
  static std::once_flag once[64];
  static cudaError_t attr_err[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::call_once(once[dev], [&] {
    attr_err[dev] = cudaFuncSetAttribute(k_decode_gemv<kTall, CB>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kDecSmemMax));
  });
  if (attr_err[dev] != cudaSuccess) return attr_err[dev];
  return cudaLaunchKernelEx(&cfg, k_decode_gemv<kTall, CB>, a);
}

// The set-up kernel, then the main kernel as its programmatic dependent.
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
  a.cps = p.cps;
  a.xs_tok = p.xs_tok;
  a.xs_bytes = static_cast<int>(s.M) * p.xs_tok;
  a.part = reinterpret_cast<float*>(scratch);
  a.T = reinterpret_cast<float*>(scratch + part_bytes(p, s));
  a.counters = reinterpret_cast<int*>(scratch + part_bytes(p, s) + t_bytes(s));
  a.t_count = a.counters + p.row_groups;
  a.err = device_error_word();
  a.T_save = T_save;
  a.Y = Y;
  if (!a.err) return QLORA_ERR_CUDA;
  note_launches(2);  // the set-up kernel and the main kernel
  const int mr = static_cast<int>(s.M) * s.r;
  const int prep_ctas = std::max(1, std::min(num_sms(), (p.row_groups + 2047) / 2048));
  cudaError_t e;
  {
    cudaLaunchConfig_t pc = {};
    pc.gridDim = dim3(static_cast<unsigned>(prep_ctas));
    pc.blockDim = dim3(256);
    pc.stream = st;
    cudaLaunchAttribute pa[1];
    pa[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pa[0].val.programmaticStreamSerializationAllowed = 1;
    pc.attrs = pa;
    pc.numAttrs = 1;
    e = cudaLaunchKernelEx(&pc, k_decode_prep, a.T, mr, a.counters, p.row_groups, a.t_count);
  }
  if (e != cudaSuccess) return cuda_status(e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.splits * p.cps));
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = dec_smem_bytes(a.xs_bytes, s.r);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (w.codebook == 1)
    e = s.M > 8 ? launch_gemv<true, 1>(cfg, a) : launch_gemv<false, 1>(cfg, a);
  else
    e = s.M > 8 ? launch_gemv<true, 0>(cfg, a) : launch_gemv<false, 0>(cfg, a);
  if (e != cudaSuccess) return cuda_status(e);
  return QLORA_OK;
}

}  // namespace

size_t decode_workspace(const LinearShape& s) {
  const DecodePlan p = plan_decode(s);
  return p.splits ? decode_scratch_bytes(p, s) + 256 : 0;
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
// keeps the split partial sums, T and the arrival counters in the fixed array below,
// which every GPU that loads this library holds until the process exits.
namespace qlora {
namespace {

constexpr size_t kStaticScratchBytes = size_t{4} << 20;  // 4 MiB per device
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

constexpr int kMaxScratchDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxScratchDevices] = {};
CUcontext g_scratch_ctx[kMaxScratchDevices] = {};

// The driver's cuCtxGetCurrent, to notice a new context on a device (after a device reset
// the array lives at a new address).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of g_decode_scratch on the current device. In host code the name
// g_decode_scratch is only a host-side stand-in, so the address is looked up with the
// device current, once per device and context, and cached.
qlora_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  if (dev < 0 || dev >= kMaxScratchDevices) {
    set_last_error("device index out of range for the static scratch table");
    return QLORA_ERR_INVALID_ARG;
  }
  CUcontext ctx = nullptr;
  if (auto fn = ctx_get_current()) fn(&ctx);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev] || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return cuda_status(e);
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_addr[dev];
  return QLORA_OK;
}

}  // namespace
}  // namespace qlora

extern "C" qlora_status qlora_linear_fwd_decode_static(const uint16_t* X, int64_t M,
                                                       qlora_nf4_weight w, const uint16_t* A,
                                                       const uint16_t* B, int r, float scale,
                                                       uint16_t* Y, float* T_save, void* stream) {
  using namespace qlora;
  // the argument checks of qlora_linear_fwd, in the same order
  qlora_status q = check_linear(M, w, r, scale);
  if (q != QLORA_OK) return q;
  if (M > kDecodeMaxM) {
    set_last_error("qlora_linear_fwd_decode_static serves 0 <= M <= 16 tokens");
    return QLORA_ERR_SHAPE;
  }
  if (M == 0) return QLORA_OK;
  if (!X || !A || !B || !Y) return QLORA_ERR_INVALID_ARG;
  if (!is_aligned16(X) || !is_aligned16(A) || !is_aligned16(B) || !is_aligned16(Y) ||
      (T_save && !is_aligned16(T_save)))
    return QLORA_ERR_ALIGN;
  const LinearShape s{M, w.n_out, w.k_in, r, scale};
  const DecodePlan p = plan_decode(s, kStaticScratchBytes);
  if (p.splits == 0) {
    char msg[200];
    std::snprintf(msg, sizeof(msg),
                  "qlora_linear_fwd_decode_static: the partial sums of %lld x %lld at M = %lld "
                  "need more than the %zu bytes of the static scratch",
                  static_cast<long long>(w.n_out), static_cast<long long>(w.k_in),
                  static_cast<long long>(M), kStaticScratchBytes);
    set_last_error(msg);
    return QLORA_ERR_WORKSPACE;
  }
  q = check_device();
  if (q != QLORA_OK) return q;
  void* scratch = nullptr;
  q = scratch_address(&scratch);
  if (q != QLORA_OK) return q;
  // Every partial sum is written before it is read, and the set-up kernel of the call
  // clears T and the arrival counters, so nothing an earlier call left in the array
  // matters.
  return launch_decode(X, w, A, B, s, p, Y, T_save, static_cast<char*>(scratch),
                       static_cast<cudaStream_t>(stream));
}
