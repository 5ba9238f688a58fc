// tables.cpp -- the NF4 and FP8 (E4M3) code tables and the exact decision thresholds
// of their nearest-entry searches. Host code only.
//
// NF4 (page "QLoRA", itwiki.kr, section "4비트 NormalFloat(NF4)"): the 16 levels are
// N(0,1) quantiles at evenly spaced probabilities between 0.9677083 and 1/2 (8 on the
// positive side, 7 on the negative side, one shared exact zero), divided by the
// largest magnitude and rounded to fp32. The fp32 bit patterns are stored below as
// data.
//
// T8 (same page, section "이중 양자화"): the 8-bit float of the double quantization,
// read as OCP FP8 E4M3; T8 = the 253 distinct finite E4M3 values divided by 448 in
// fp32, ascending.
//
// Thresholds: the quantizer picks argmin_i fl32(|x - table_i|), first index on ties.
// For every x in [-1, 1] this index is a non-decreasing function of x (each distance
// is a monotone function of x and the table entries are further apart than one ulp
// of any |x - t| <= 2), so it equals the number of thresholds <= x, where threshold
// i is the smallest fp32 x whose index exceeds i. They are found here by bisection
// over the ordered fp32 bit patterns, evaluating the argmin rule itself.
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <limits>
#include <mutex>

#include "internal.h"

namespace qlora {

const uint32_t kNf4Bits[16] = {
    0xbf800000u, 0xbf3239b3u, 0xbf066b30u, 0xbeca32a0u, 0xbe91a24cu, 0xbe3d353fu,
    0xbdba786bu, 0x00000000u, 0x3da2fb03u, 0x3e24cae1u, 0x3e7c04dcu, 0x3ead0338u,
    0x3ee1a4b7u, 0x3f1007aau, 0x3f3913b1u, 0x3f800000u};

// The comparison codebook of the same section: 16 evenly spaced levels on [-1, 1]
// (-1 + 2i/15 in double, the end point exact, rounded to fp32).
const uint32_t kUniform4Bits[16] = {
    0xbf800000u, 0xbf5ddddeu, 0xbf3bbbbcu, 0xbf19999au, 0xbeeeeeefu, 0xbeaaaaabu,
    0xbe4ccccdu, 0xbd888889u, 0x3d888889u, 0x3e4ccccdu, 0x3eaaaaabu, 0x3eeeeeefu,
    0x3f19999au, 0x3f3bbbbcu, 0x3f5ddddeu, 0x3f800000u};

namespace {

float bits_to_float(uint32_t u) {
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}
uint32_t float_to_bits(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return u;
}
// Monotone map from fp32 (finite) to uint32: a < b  <=>  key(a) < key(b); -0 < +0.
uint32_t order_key(float f) {
  const uint32_t u = float_to_bits(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
float from_order_key(uint32_t k) {
  const uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return bits_to_float(u);
}

// argmin_i fl32(|x - t_i|), lowest index on ties. volatile keeps each difference an
// fp32 operation.
int nearest_index(float x, const float* t, int n) {
  int best = 0;
  volatile float bd = std::fabs(x - t[0]);
  for (int i = 1; i < n; ++i) {
    volatile float d = std::fabs(x - t[i]);
    if (d < bd) {
      bd = d;
      best = i;
    }
  }
  return best;
}

// Smallest fp32 x in (t[i], t[i+1]] whose nearest index is > i.
float first_above(const float* t, int n, int i) {
  uint32_t lo = order_key(t[i]);      // nearest index == i here
  uint32_t hi = order_key(t[i + 1]);  // nearest index == i + 1 here
  while (hi - lo > 1) {
    const uint32_t mid = lo + (hi - lo) / 2;
    if (nearest_index(from_order_key(mid), t, n) > i)
      hi = mid;
    else
      lo = mid;
  }
  return from_order_key(hi);
}

float e4m3_value(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  const float v = (e == 0) ? std::ldexp(static_cast<float>(m), -9)
                           : std::ldexp(static_cast<float>(8u + m), static_cast<int>(e) - 10);
  return (b & 0x80u) ? -v : v;
}

struct CodebookTables {
  float levels[16];
  Nf4Thresholds thr;
  Nf4BucketTable buckets;
};

// Thresholds and the bucket table of one 16-level codebook.
void build_codebook(const uint32_t (&bits)[16], CodebookTables& cb) {
  for (int i = 0; i < 16; ++i) cb.levels[i] = bits_to_float(bits[i]);
  for (int i = 0; i < 15; ++i) cb.thr.t[i] = first_above(cb.levels, 16, i);
  // Bucket b holds the fp32 x with round-half-even(S x + S) == b (S = kBucketScale): its
  // edges are (2b -+ 1 - 2S) / 2S, each tie going to the even bucket.
  const double s2 = 2.0 * kBucketScale;
  for (int b = 0; b < kCodeBuckets; ++b) {
    float xmin = static_cast<float>((2.0 * b - 1.0 - s2) / s2);
    float xmax = static_cast<float>((2.0 * b + 1.0 - s2) / s2);
    if (b & 1) {
      xmin = std::nextafter(xmin, std::numeric_limits<float>::infinity());
      xmax = std::nextafter(xmax, -std::numeric_limits<float>::infinity());
    }
    int code = 0;
    for (int i = 0; i < 15; ++i) code += (xmin >= cb.thr.t[i]) ? 1 : 0;
    float thr = std::numeric_limits<float>::infinity();
    int inside = 0;
    for (int i = 0; i < 15; ++i)
      if (cb.thr.t[i] > xmin && cb.thr.t[i] <= xmax) {
        thr = cb.thr.t[i];
        ++inside;
      }
    if (inside > 1) std::abort();  // the table form needs at most one threshold per bucket
    cb.buckets.thr[b] = thr;
    cb.buckets.code[b] = static_cast<uint8_t>(code);
  }
}

struct Tables {
  CodebookTables cb[kCodebooks];
  T8Thresholds t8;
  float t8_vals[kT8Size];
  uint8_t t8_code[kT8Size];
};

const Tables& tables() {
  static Tables tab;
  static std::once_flag once;
  std::call_once(once, [] {
    build_codebook(kNf4Bits, tab.cb[0]);
    build_codebook(kUniform4Bits, tab.cb[1]);
    // T8 in ascending order: -448 .. -min (0xFE .. 0x81), 0 (0x00), +min .. +448.
    int n = 0;
    for (int b = 0xFE; b >= 0x81; --b) tab.t8_code[n++] = static_cast<uint8_t>(b);
    tab.t8_code[n++] = 0x00;
    for (int b = 0x01; b <= 0x7E; ++b) tab.t8_code[n++] = static_cast<uint8_t>(b);
    for (int i = 0; i < kT8Size; ++i) {
      volatile float v = e4m3_value(tab.t8_code[i]);
      volatile float q = v / 448.0f;
      tab.t8_vals[i] = q;
    }
    for (int i = 0; i < kT8Size - 1; ++i) tab.t8.t[i] = first_above(tab.t8_vals, kT8Size, i);
  });
  return tab;
}

}  // namespace

const Nf4Thresholds& nf4_thresholds() { return tables().cb[0].thr; }
const Nf4BucketTable& code_buckets(int codebook) { return tables().cb[codebook].buckets; }
const float* codebook_levels(int codebook) { return tables().cb[codebook].levels; }
const T8Thresholds& t8_thresholds() { return tables().t8; }
const float* t8_values() { return tables().t8_vals; }
const uint8_t* t8_codes() { return tables().t8_code; }

}  // namespace qlora

extern "C" void qlora_nf4_table(float* out16) {
  if (!out16) return;
  for (int i = 0; i < 16; ++i) std::memcpy(&out16[i], &qlora::kNf4Bits[i], 4);
}

extern "C" void qlora_nf4_thresholds(float* out15) {
  if (!out15) return;
  const auto& t = qlora::nf4_thresholds();
  for (int i = 0; i < 15; ++i) out15[i] = t.t[i];
}

extern "C" void qlora_nf4_code_buckets(float* thr33, uint8_t* code33) {
  const auto& t = qlora::code_buckets(0);
  for (int i = 0; i < qlora::kCodeBuckets; ++i) {
    if (thr33) thr33[i] = t.thr[i];
    if (code33) code33[i] = t.code[i];
  }
}

extern "C" void qlora_fp8_thresholds(float* out252, float* t8_out253, uint8_t* codes_out253) {
  const auto& t = qlora::t8_thresholds();
  if (out252)
    for (int i = 0; i < qlora::kT8Size - 1; ++i) out252[i] = t.t[i];
  if (t8_out253)
    for (int i = 0; i < qlora::kT8Size; ++i) t8_out253[i] = qlora::t8_values()[i];
  if (codes_out253)
    for (int i = 0; i < qlora::kT8Size; ++i) codes_out253[i] = qlora::t8_codes()[i];
}

extern "C" int qlora_codebook_tables(int32_t codebook, float* levels16, float* thr15,
                                     float* bucket_thr33, uint8_t* bucket_code33) {
  if (codebook < 0 || codebook >= qlora::kCodebooks) return -1;
  const auto& cb = qlora::tables().cb[codebook];
  for (int i = 0; i < 16; ++i)
    if (levels16) levels16[i] = cb.levels[i];
  for (int i = 0; i < 15; ++i)
    if (thr15) thr15[i] = cb.thr.t[i];
  for (int i = 0; i < qlora::kCodeBuckets; ++i) {
    if (bucket_thr33) bucket_thr33[i] = cb.buckets.thr[i];
    if (bucket_code33) bucket_code33[i] = cb.buckets.code[i];
  }
  return 0;
}
