// merge.cu -- merge_and_unload: W_merged = bf16(W_hat + scale (A B)^T), [N, K] bf16.
// (blog "QLoRA", irregular6612, section "학습 → 추론 파이프라인 (실무)": after training the
// base is dequantized to BF16 and the LoRA term added, with its alpha/r scale, section
// "재양자화 시 주의사항"; itwiki "QLoRA", section "한계와 주의점".)
//
// A CTA owns a band of 64 rows n and walks consecutive 64 x 64 tiles (one 64-block of K
// per row each) along K. The rank-r
// product goes through mma.sync.m16n8k16 (bf16 in, fp32 accumulation) with ldmatrix
// fragments from shared memory: at r = 64 it is 64 multiply-adds per output element, more
// than the CUDA cores sustain at the 2.5 bytes of HBM traffic each element costs. Every
// output element is then fma(scale, product, W_hat) in fp32 (W_hat the exact double
// dequantization, a bf16 value), rounded to bf16, and the tile leaves through shared
// memory in 16-byte stores.
#include <cuda_bf16.h>

#include "internal.h"
#include "nf4_device.cuh"

namespace qlora {
namespace {

constexpr int kMergeTile = 64;
constexpr int kMergeThreads = 256;  // 8 warps: 16 rows x 32 columns of the tile each
constexpr int kRowPad = 72;         // shared rows of 64 bf16 + 8: 16-byte aligned, banks spread

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

struct MergeArgs {
  const uint8_t* codes;
  const uint8_t* c2;
  const float* c1;
  const float* mean;
  const uint16_t* A;  // [K, r]
  const uint16_t* B;  // [r, N]
  int64_t N, K;
  int r;
  float scale;
  uint16_t* out;      // [N, K]
};

// grid: x = 64-row bands of W, y = groups of `ktiles` consecutive 64-column tiles. B's
// band, the T8 table and the MMA fragments that come from B are staged once per CTA.
template <int CB>
__global__ void __launch_bounds__(kMergeThreads) k_merge_lora(const MergeArgs a, int ktiles) {
  __shared__ __align__(16) uint16_t bs[kMergeTile][kRowPad];  // B[j][n0 + i] (rows j >= r zero)
  __shared__ __align__(16) uint16_t as[kMergeTile][kRowPad];  // A[k0 + i][j] (cols j >= r zero)
  __shared__ __align__(16) uint16_t os[kMergeTile][kRowPad];  // output tile [n][k]
  __shared__ __align__(16) uint8_t cs[kMergeTile][32];        // codes of the tile's rows
  __shared__ float srow[kMergeTile];                          // block scale of each row
  __shared__ float lut[16];
  __shared__ float t8[256];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wr = 16 * (warp & 3);   // first tile row of this warp
  const int wc = 32 * (warp >> 2);  // first tile column of this warp
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kMergeTile;
  const int64_t kt_total = a.K / kMergeTile;
  const int64_t kt0 = static_cast<int64_t>(blockIdx.y) * ktiles;
  const int64_t kt1 = kt0 + ktiles < kt_total ? kt0 + ktiles : kt_total;
  const int r = a.r, r16 = (a.r + 15) & ~15;
  const float mean = *a.mean;

  for (int e = tid; e < 256; e += kMergeThreads) t8[e] = t8_value(e);
  if (tid < 16) lut[tid] = code_level<CB>(tid);
  for (int idx = tid; idx < r16 * 8; idx += kMergeThreads) {
    const int j = idx >> 3, c = idx & 7;  // chunk c of row j: columns n0 + 8c .. + 7
    const int64_t n = n0 + c * 8;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (j < r && n < a.N) v = __ldg(reinterpret_cast<const uint4*>(a.B + j * a.N + n));
    *reinterpret_cast<uint4*>(&bs[j][c * 8]) = v;
  }
  __syncthreads();
  // the math A operand of the rank-r product is B^T (rows n, columns j), read transposed
  // from bs[j][n]: the same for every column tile, so it stays in registers
  const int mat = lane >> 3, rr = lane & 7;
  uint32_t af[4][4];
#pragma unroll
  for (int jb = 0; jb < 4; ++jb)
    if (16 * jb < r16)
      ldsm_x4_trans(af[jb], &bs[16 * jb + rr + ((mat >> 1) << 3)][wr + ((mat & 1) << 3)]);
  const int g = lane >> 2, t = lane & 3;

  for (int64_t kt = kt0; kt < kt1; ++kt) {
    const int64_t k0 = kt * kMergeTile;
    const uint16_t* arow = a.A + k0 * r;
#pragma unroll
    for (int it = 0; it < (kMergeTile * 8) / kMergeThreads; ++it) {
      const int idx = tid + it * kMergeThreads;
      const int i = idx >> 3, c = idx & 7;  // 8-wide chunk c of row k0 + i (zeros past r)
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (c * 8 < r) v = __ldg(reinterpret_cast<const uint4*>(arow + i * r + c * 8));
      *reinterpret_cast<uint4*>(&as[i][c * 8]) = v;
    }
    if (tid < 2 * kMergeTile) {
      const int i = tid >> 1, h = tid & 1;  // 16 code bytes of row n0 + i
      const int64_t n = n0 + i;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (n < a.N)
        v = __ldg(reinterpret_cast<const uint4*>(a.codes + n * (a.K / 2) + k0 / 2 + h * 16));
      *reinterpret_cast<uint4*>(&cs[i][h * 16]) = v;
    } else if (tid < 3 * kMergeTile) {
      const int i = tid - 2 * kMergeTile;
      const int64_t n = n0 + i;
      float sv = 0.f;
      if (n < a.N) {
        const int64_t j = n * (a.K / 64) + kt;
        sv = block_scale_tab(t8, __ldg(a.c2 + j), __ldg(a.c1 + (j >> 8)), mean);
      }
      srow[i] = sv;
    }
    __syncthreads();

    // (A B)^T for this warp's 16 rows and 32 columns: the math B operand (j x k) is A^T,
    // whose columns are the rows of as
    float acc[4][4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[q][i] = 0.f;
#pragma unroll
    for (int jb = 0; jb < 4; ++jb) {
      if (16 * jb >= r16) break;
#pragma unroll
      for (int kt2 = 0; kt2 < 2; ++kt2) {
        uint32_t bf[4];
        ldsm_x4(bf, &as[wc + 16 * kt2 + rr + ((mat >> 1) << 3)][16 * jb + ((mat & 1) << 3)]);
        mma_16816(acc[2 * kt2], af[jb], bf[0], bf[1]);
        mma_16816(acc[2 * kt2 + 1], af[jb], bf[2], bf[3]);
      }
    }

    // C fragment: (row g, columns 2t, 2t+1) and (row g + 8, same columns) of each 8-column tile
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int nl = wr + g + 8 * h;
        const int kl = wc + 8 * q + 2 * t;
        const uint32_t byte = cs[nl][kl >> 1];  // codes of columns kl (low nibble), kl + 1
        const float sv = srow[nl];
        const float w0 =
            __uint_as_float(static_cast<uint32_t>(bf16_bits_rn(__fmul_rn(lut[byte & 15u], sv))) << 16);
        const float w1 =
            __uint_as_float(static_cast<uint32_t>(bf16_bits_rn(__fmul_rn(lut[byte >> 4], sv))) << 16);
        const uint32_t y0 = bf16_bits_rn(__fmaf_rn(a.scale, acc[q][2 * h], w0));
        const uint32_t y1 = bf16_bits_rn(__fmaf_rn(a.scale, acc[q][2 * h + 1], w1));
        *reinterpret_cast<uint32_t*>(&os[nl][kl]) = y0 | (y1 << 16);
      }
    __syncthreads();  // os complete; as, cs and srow free for the next tile
#pragma unroll
    for (int i = 0; i < (kMergeTile * 8) / kMergeThreads; ++i) {
      const int idx = tid + i * kMergeThreads;
      const int row = idx >> 3, ch = idx & 7;
      const int64_t n = n0 + row;
      if (n < a.N)
        *reinterpret_cast<uint4*>(a.out + n * a.K + k0 + ch * 8) =
            *reinterpret_cast<const uint4*>(&os[row][ch * 8]);
    }
  }
}

}  // namespace

cudaError_t launch_merge_lora(const qlora_nf4_weight& w, const uint16_t* A, const uint16_t* B,
                              int r, float scale, uint16_t* out, cudaStream_t st) {
  MergeArgs a;
  a.codes = w.codes;
  a.c2 = w.c2;
  a.c1 = w.c1;
  a.mean = w.mean;
  a.A = A;
  a.B = B;
  a.N = w.n_out;
  a.K = w.k_in;
  a.r = r;
  a.scale = scale;
  a.out = out;
  // enough CTAs for several waves, each walking at most 8 column tiles of its band
  const int64_t bands = (w.n_out + kMergeTile - 1) / kMergeTile;
  const int64_t kt_total = w.k_in / kMergeTile;
  const int64_t want = static_cast<int64_t>(num_sms()) * 24;
  int64_t ktiles = (bands * kt_total + want - 1) / want;
  ktiles = ktiles < 1 ? 1 : (ktiles > 8 ? 8 : ktiles);
  if ((kt_total + ktiles - 1) / ktiles > 65535) ktiles = (kt_total + 65534) / 65535;  // grid y
  const dim3 grid(static_cast<unsigned>(bands),
                  static_cast<unsigned>((kt_total + ktiles - 1) / ktiles));
  auto kern = w.codebook == 1 ? k_merge_lora<1> : k_merge_lora<0>;
  note_launches(1);
  kern<<<grid, kMergeThreads, 0, st>>>(a, static_cast<int>(ktiles));
  return cudaGetLastError();
}

}  // namespace qlora
