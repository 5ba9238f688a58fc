// nf4_device.cuh -- device-side pieces of the double dequantization shared by the
// standalone dequant, the fused GEMM, the decode and the merge kernels (NF4 is the
// codebook L below unless a kernel is instantiated for the uniform one):
//   s_j   = fl32(fl32(T8[c2_j] * c1[j / 256]) + mean)     (T8[e] = fl32(e4m3(e) / 448))
//   W_hat = bf16_rn(fl32(NF4[code] * s_j))
// (page "QLoRA", itwiki.kr: sections "4비트 NormalFloat(NF4)" and "이중 양자화", and
// doubleDequant in section "계산 방식").
#pragma once

#include <cstdint>

#include "sm100.cuh"

namespace qlora {

// Level i of codebook CB as an fp32 constant (bit patterns, ascending): CB 0 is NF4,
// CB 1 the evenly spaced comparison codebook of the same section (-1 + 2i/15).
template <int CB>
__device__ __forceinline__ float code_level(int i) {
  constexpr uint32_t nf4[16] = {0xbf800000u, 0xbf3239b3u, 0xbf066b30u, 0xbeca32a0u,
                                0xbe91a24cu, 0xbe3d353fu, 0xbdba786bu, 0x00000000u,
                                0x3da2fb03u, 0x3e24cae1u, 0x3e7c04dcu, 0x3ead0338u,
                                0x3ee1a4b7u, 0x3f1007aau, 0x3f3913b1u, 0x3f800000u};
  constexpr uint32_t uni[16] = {0xbf800000u, 0xbf5ddddeu, 0xbf3bbbbcu, 0xbf19999au,
                                0xbeeeeeefu, 0xbeaaaaabu, 0xbe4ccccdu, 0xbd888889u,
                                0x3d888889u, 0x3e4ccccdu, 0x3eaaaaabu, 0x3eeeeeefu,
                                0x3f19999au, 0x3f3bbbbcu, 0x3f5ddddeu, 0x3f800000u};
  return __uint_as_float(CB == 0 ? nf4[i] : uni[i]);
}
__device__ __forceinline__ float nf4_level(int i) { return code_level<0>(i); }

// code_level for an index only known at run time, through selects over the constant
// levels (an indexed local array would live in local memory).
template <int CB>
__device__ __forceinline__ float code_level_rt(int i) {
  float v = 0.f;
#pragma unroll
  for (int j = 0; j < 16; ++j)
    if (i == j) v = code_level<CB>(j);
  return v;
}

// Value of an OCP FP8 E4M3 bit pattern (exact in fp32).
__device__ __forceinline__ float e4m3_value(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  const float v = (e == 0u) ? static_cast<float>(m) * 0.001953125f  // m * 2^-9
                            : __uint_as_float(((e + 120u) << 23) | (m << 20));
  return (b & 0x80u) ? -v : v;
}

// T8 entry of an E4M3 code: fl32(e4m3 / 448) (IEEE division).
__device__ __forceinline__ float t8_value(uint32_t c2) {
  return __fdiv_rn(e4m3_value(c2), 448.0f);
}

// Reconstructed absmax of one 64-block from its double-quantized constants.
__device__ __forceinline__ float block_scale(uint32_t c2, float c1, float mean) {
  return __fadd_rn(__fmul_rn(t8_value(c2), c1), mean);
}

// The same with T8 read from a 256-entry table (t8[e] = t8_value(e)).
__device__ __forceinline__ float block_scale_tab(const float* t8, uint32_t c2, float c1,
                                                 float mean) {
  return __fadd_rn(__fmul_rn(t8[c2], c1), mean);
}

// 16-entry bf16 table {bf16(NF4[i] * s)} split into byte planes for prmt lookups:
// lo[q] holds the low bytes of entries 4q..4q+3, hi[q] their high bytes.
struct Nf4Lut {
  uint32_t lo[4];
  uint32_t hi[4];
};

template <int CB = 0>
__device__ __forceinline__ void build_lut(float s, Nf4Lut& t) {
  uint32_t p[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    p[i] = pack_bf16x2_rn(__fmul_rn(code_level<CB>(2 * i), s), __fmul_rn(code_level<CB>(2 * i + 1), s));
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    t.lo[q] = prmt(p[2 * q], p[2 * q + 1], 0x6420u);
    t.hi[q] = prmt(p[2 * q], p[2 * q + 1], 0x7531u);
  }
}

// Eight 4-bit codes (nibble i of w = code of element i) -> four bf16x2 registers
// o[i] = (element 2i in the low half, element 2i+1 in the high half).
// The raw codes serve as prmt selectors: bits 0-2 index a byte of an 8-byte window
// (entries 0-7, or entries 8-15 with bit 3 flipped), and a selector whose bit 3 is set
// replicates a sign bit instead of copying, which only happens in the window that the
// byte mask then discards. The mask itself is a sign replication too: byte j of w has
// bit 3 of code 2j+1 as its sign bit, byte j of w << 4 that of code 2j.
__device__ __forceinline__ void lut_decode8(uint32_t w, const Nf4Lut& t, uint32_t (&o)[4]) {
  const uint32_t w4 = w << 4;
  const uint32_t wx = w ^ 0x88888888u;  // selectors into entries 8-15
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t s = h ? (w >> 16) : w;
    const uint32_t sx = h ? (wx >> 16) : wx;
    const uint32_t mask = prmt(w, w4, h ? 0xBFAEu : 0x9D8Cu);  // 0xFF where the code is >= 8
    const uint32_t lo = (prmt(t.lo[0], t.lo[1], s) & ~mask) | (prmt(t.lo[2], t.lo[3], sx) & mask);
    const uint32_t hi = (prmt(t.hi[0], t.hi[1], s) & ~mask) | (prmt(t.hi[2], t.hi[3], sx) & mask);
    o[2 * h] = prmt(lo, hi, 0x5140u);
    o[2 * h + 1] = prmt(lo, hi, 0x7362u);
  }
}

// ---- T8, the 8-bit float code table of the double quantization: the 253 distinct finite
// E4M3 values / 448 in ascending order (page "QLoRA", itwiki.kr, section "이중 양자화").
constexpr int kT8Entries = 253;

// Index of entry i of T8 -> its E4M3 bit pattern.
__device__ __forceinline__ uint32_t t8_index_to_code(int i) {
  return (i < 126) ? (0xFEu - static_cast<uint32_t>(i)) : (i == 126 ? 0u : static_cast<uint32_t>(i - 126));
}
// E4M3 bit pattern -> index of its value in T8 (both zeros -> the one zero entry, 126).
__device__ __forceinline__ int t8_code_to_index(uint32_t e) {
  return (e & 0x80u) ? static_cast<int>(0xFEu - e) : static_cast<int>(126u + e);
}
// E4M3 bit patterns of two fp32 values (hardware conversion, round to nearest even,
// saturated at +-448): lo in bits 0-7, hi in bits 8-15.
__device__ __forceinline__ uint32_t e4m3x2_rn(float lo, float hi) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  return d;
}

// The nearest-entry search over T8 by E4M3 code: for each code c the threshold just
// above its entry (up), the one just below (dn), and the codes of the next and previous
// entries and of the entry itself (moves: bits 0-7 next, 8-15 previous, 16-23 self; the
// negative zero's self is the zero code). Built in shared memory by every CTA from the
// 252 exact decision thresholds (build_t8_search).
struct T8Search {
  float up[256];
  float dn[256];
  uint32_t moves[256];
};

// Fill t from sth (sth[k] = the smallest fp32 whose nearest T8 entry is k + 1) with the
// CTA's threads; the caller synchronises before use.
__device__ __forceinline__ void build_t8_search(const float* sth, T8Search& t) {
  for (int c = threadIdx.x; c < 256; c += blockDim.x) {
    const uint32_t e = static_cast<uint32_t>(c);
    const bool nan = (e & 0x7Fu) == 0x7Fu;  // never produced by a saturating conversion
    const int i = nan ? 126 : t8_code_to_index(e);
    t.up[c] = i < kT8Entries - 1 ? sth[i] : __int_as_float(0x7F800000);   // +inf
    t.dn[c] = i > 0 ? sth[i - 1] : __int_as_float(0xFF800000);             // -inf
    const uint32_t next = t8_index_to_code(i < kT8Entries - 1 ? i + 1 : i);
    const uint32_t prev = t8_index_to_code(i > 0 ? i - 1 : i);
    t.moves[c] = next | (prev << 8) | (t8_index_to_code(i) << 16);
  }
}

// E4M3 codes of the nearest T8 entries (ties to the lower index) of y0 and y1 in [-1, 1]:
// code of y0 in bits 0-7, of y1 in bits 8-15. The answer is the number of decision
// thresholds <= y. The hardware E4M3 conversion of fl32(448 y) gives a candidate entry:
// its rounding errors are below 2^-23 relative while neighbouring E4M3 values lie at
// least 1/16 apart, so the answer is the candidate or one of its two neighbours, and one
// comparison with each of the two thresholds around the candidate decides it.
// This form reads the 252 thresholds sth directly (no table to build: for kernels whose
// CTAs code few values); the T8Search form below needs fewer instructions per value.
__device__ __forceinline__ uint32_t t8_nearest_codes2(float y0, float y1, const float* sth) {
  const uint32_t cand = e4m3x2_rn(__fmul_rn(y0, 448.0f), __fmul_rn(y1, 448.0f));
  uint32_t out = 0u;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float y = h ? y1 : y0;
    const int c = t8_code_to_index((cand >> (8 * h)) & 0xFFu);
    const float up = sth[min(c, kT8Entries - 2)];  // threshold between entries c and c + 1
    const float dn = sth[max(c - 1, 0)];           // threshold between entries c - 1 and c
    const int pos = c + ((c < kT8Entries - 1 && y >= up) ? 1 : 0) - ((c > 0 && y < dn) ? 1 : 0);
    out |= t8_index_to_code(pos) << (8 * h);
  }
  return out;
}
__device__ __forceinline__ uint32_t t8_nearest_codes2(float y0, float y1, const T8Search& t) {
  const uint32_t cand = e4m3x2_rn(__fmul_rn(y0, 448.0f), __fmul_rn(y1, 448.0f));
  uint32_t out = 0u;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float y = h ? y1 : y0;
    const uint32_t c = (cand >> (8 * h)) & 0xFFu;
    const uint32_t mv = t.moves[c];
    const uint32_t sh = y >= t.up[c] ? 0u : (y < t.dn[c] ? 8u : 16u);
    out |= ((mv >> sh) & 0xFFu) << (8 * h);
  }
  return out;
}

__device__ __forceinline__ uint16_t bf16_bits_rn(float x) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %1;" : "=r"(d) : "f"(x));
  return static_cast<uint16_t>(d & 0xFFFFu);
}

}  // namespace qlora
