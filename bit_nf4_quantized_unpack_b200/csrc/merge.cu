// merge.cu -- merge_and_unload: W_merged = bf16(W_hat + scale (A B)^T), [N, K] bf16.
// (blog "QLoRA", irregular6612, section "학습 → 추론 파이프라인 (실무)": after training the
// base is dequantized to BF16 and the LoRA term added, with its alpha/r scale, section
// "재양자화 시 주의사항"; itwiki "QLoRA", section "한계와 주의점".)
//
// Persistent tcgen05 kernel (two CTAs per SM) over tiles of 128 rows n x 128 columns k:
//   warp 0      TMA: B's 128 columns n (B [r, N] as an MN-major operand, two 64-wide
//               chunks), A's 128 rows k (A [K, r], K-major over j) and the tile's codes
//               (128 rows x 64 bytes), into one of two stages
//   warp 1      MMA: ceil(r/16) tcgen05.mma of 128 x 128 x 16 into one of two 128-column
//               TMEM buffers, D[n][k] = sum_j B[j][n] A[k][j] in fp32
//   warps 2-9   epilogue, two per TMEM lane quarter (one 64-column block each): the row's
//               64 codes and block constants are expanded exactly through a prmt table of
//               the block's 16 bf16 levels, and every element becomes
//               bf16(fma(scale, D, W_hat)); each 32 x 32 chunk is staged in shared memory
//               (64-byte swizzle) and leaves with one TMA tile store
// At r = 64 the rank-r product is 64 multiply-adds per output element, which the tensor
// cores absorb; the next tile's product runs while the epilogue drains this one.
#include <cuda.h>
#include <cuda_bf16.h>

#include "internal.h"
#include "nf4_device.cuh"

namespace qlora {
namespace {

constexpr int kMgRows = 128;                     // rows n of a tile (TMEM lanes)
constexpr int kMgCols = 128;                     // columns k of a tile (TMEM columns)
constexpr int kMgStages = 2;
constexpr uint32_t kMgABytes = kMgCols * 64 * 2;  // A rows k x 64 j (zero past r)
constexpr uint32_t kMgBBytes = kMgRows * 64 * 2;  // B columns n x 64 j, two MN-major chunks
constexpr int kMgEpiWarps = 8;
constexpr int kMgThreads = 32 * (2 + kMgEpiWarps);
constexpr uint32_t kMgCBytes = kMgRows * kMgCols / 2;  // the tile's codes, 64-byte swizzle
constexpr uint32_t kMgStageOut = 32 * 64;       // per epilogue warp: one 32 x 32 bf16 chunk
constexpr uint32_t kMgSmem = kMgStages * (kMgABytes + kMgBBytes + kMgCBytes) +
                             kMgEpiWarps * kMgStageOut + 1024 + 256 + 1024;
constexpr int kMgCtasPerSm = 2;  // TMEM: 2 x (2 x kMgCols) columns

struct MergeArgs {
  const uint8_t* c2;
  const float* c1;
  const float* mean;
  int64_t N, K;
  int r;
  float scale;
  uint16_t* out;   // [N, K]
  int row_tiles;   // tiles along n
  int num_tiles;   // row_tiles x tiles along k
  int* err;
};

template <int CB>
__global__ void __launch_bounds__(kMgThreads, kMgCtasPerSm)
    k_merge_lora(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                 const __grid_constant__ CUtensorMap tm_codes,
                 const __grid_constant__ CUtensorMap tm_out, const MergeArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* a_s = smem;                                   // [stages][kMgABytes]
  uint8_t* b_s = a_s + kMgStages * kMgABytes;            // [stages][kMgBBytes]
  uint8_t* c_s = b_s + kMgStages * kMgBBytes;             // [stages][128 rows][64 B] codes
  uint8_t* o_s = c_s + kMgStages * kMgCBytes;             // [epilogue warps][32][64 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(o_s + kMgEpiWarps * kMgStageOut);
  uint64_t* full = bars;                    // [stages] operands landed
  uint64_t* empty = full + kMgStages;       // [stages] MMAs and epilogue warps done with them
  uint64_t* acc_full = empty + kMgStages;   // [2] product complete
  uint64_t* acc_empty = acc_full + 2;       // [2] product read out
  uint64_t* mma_drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* t8 = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 256);  // [256]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < 256; e += blockDim.x) t8[e] = t8_value(e);
  const int my_tiles = (static_cast<int>(blockIdx.x) < args.num_tiles)
                           ? (args.num_tiles - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1
                           : 0;
  // consecutive CTAs take consecutive row bands of the same columns (A tile shared in L2)
  auto tile_coords = [&](int i, int64_t& n0, int64_t& k0) {
    const int tile = blockIdx.x + i * gridDim.x;
    n0 = static_cast<int64_t>(tile % args.row_tiles) * kMgRows;
    k0 = static_cast<int64_t>(tile / args.row_tiles) * kMgCols;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMgStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + kMgEpiWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kMgEpiWarps);
    }
    mbar_init(mma_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * kMgCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------ TMA
    if (lane == 0) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      tma_prefetch_desc(&tm_codes);
      int issued = 0;
      for (int i = 0; i < my_tiles; ++i) {
        const int s = i % kMgStages;
        if (i >= kMgStages && !mbar_wait(&empty[s], ((i / kMgStages) - 1) & 1u, abort_flag)) {
          record_error(args.err, abort_flag, kErrTimeoutProducer);
          break;
        }
        int64_t n0, k0;
        tile_coords(i, n0, k0);
        mbar_arrive_expect_tx(&full[s], kMgABytes + kMgBBytes + kMgCBytes);
        tma_load_2d(c_s + s * kMgCBytes, &tm_codes, &full[s], static_cast<int>(k0 / 2),
                    static_cast<int>(n0));
        tma_load_2d(b_s + s * kMgBBytes, &tm_b, &full[s], static_cast<int>(n0), 0);
        tma_load_2d(b_s + s * kMgBBytes + 8192, &tm_b, &full[s], static_cast<int>(n0) + 64, 0);
        tma_load_2d(a_s + s * kMgABytes, &tm_a, &full[s], 0, static_cast<int>(k0));
        ++issued;
      }
      if (*abort_flag)  // copies in flight land before the CTA exits
        for (int i = (issued > kMgStages ? issued - kMgStages : 0); i < issued; ++i)
          mbar_wait_drain(&full[i % kMgStages], (i / kMgStages) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      // A operand: B^T (rows n, K = j) MN-major, 64-row chunks 8 KB apart; B operand: A's
      // rows k, K-major. Per 16-wide j slice the MN-major operand advances 16 rows of
      // 128 bytes (2048 B) and the K-major one 32 bytes.
      constexpr uint32_t idesc = idesc_bf16_f32(kMgRows, kMgCols, true, false);
      const int nk = (args.r + 15) / 16;
      int done = 0;
      for (int i = 0; i < my_tiles; ++i) {
        const int s = i % kMgStages, b = i & 1;
        if (!mbar_wait(&full[s], (i / kMgStages) & 1u, abort_flag)) {
          record_error(args.err, abort_flag, kErrTimeoutMma);
          break;
        }
        if (i >= 2 && !mbar_wait(&acc_empty[b], ((i >> 1) - 1) & 1u, abort_flag)) {
          record_error(args.err, abort_flag, kErrTimeoutMma);
          break;
        }
        tc_fence_after();
        const uint64_t da = smem_desc_sw128(smem_u32(b_s + s * kMgBBytes), 8192, 1024);
        const uint64_t db = smem_desc_sw128(smem_u32(a_s + s * kMgABytes), 16, 1024);
        for (int kk = 0; kk < nk; ++kk)
          umma_bf16(tmem_base + b * kMgCols, da + kk * 128u, db + kk * 2u, idesc, kk != 0);
        umma_commit(&empty[s]);
        umma_commit(&acc_full[b]);
        ++done;
      }
      umma_commit(mma_drain);
      mbar_wait_drain(mma_drain, 0);
      uint32_t par;
      for (int s = 0; s < kMgStages; ++s)
        if (last_use(done, kMgStages, s, par)) mbar_wait_drain(&empty[s], par);
      for (int b = 0; b < 2; ++b)
        if (last_use(done, 2, b, par)) mbar_wait_drain(&acc_full[b], par);
    }
  } else {
    // ------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int quarter = warp & 3;           // TMEM lanes this warp may read
    const int col0 = (ew >> 2) * 64;        // its 64-column block of the tile
    const float mean = *args.mean;
    uint8_t* stage1 = o_s + ew * kMgStageOut;  // this warp's chunk buffer
    int chunks = 0;
    if (lane == 0) tma_prefetch_desc(&tm_out);
    const int64_t bpr = args.K / 64;        // 64-blocks per row
    // the raw block constants of this thread's row in its block of tile i (the scale is
    // formed when the block is used, so the loads stay in flight meanwhile)
    auto fetch = [&](int i, uint32_t& e2, float& e1, bool& live, int64_t& n, int64_t& kb) {
      int64_t n0, k0;
      tile_coords(i, n0, k0);
      n = n0 + quarter * 32 + lane;
      kb = k0 + col0;
      e2 = 0u;
      e1 = 0.f;
      live = n < args.N && kb < args.K;
      if (live) {
        const int64_t j = n * bpr + kb / 64;
        e2 = __ldg(args.c2 + j);
        e1 = __ldg(args.c1 + (j >> 8));
      }
    };
    // this lane's row of the staged codes: its 16-byte groups g at slot g ^ ((row >> 1) & 3)
    const int crow = quarter * 32 + lane;
    const int g0 = col0 / 32;  // first 16-byte group of this warp's block
    uint32_t e2;
    float e1;
    bool live;
    int64_t n, kb;
    if (my_tiles > 0) fetch(0, e2, e1, live, n, kb);
    for (int i = 0; i < my_tiles; ++i) {
      const int b = i & 1, s = i % kMgStages;
      const float s_cur = live ? block_scale_tab(t8, e2, e1, mean) : 0.f;
      const int64_t n_cur = n, kb_cur = kb;
      if (i + 1 < my_tiles) fetch(i + 1, e2, e1, live, n, kb);  // one tile ahead
      Nf4Lut lut;
      build_lut<CB>(s_cur, lut);
      // codes of stage s (landed before the MMA that completes acc_full ran)
      if (!mbar_wait(&full[s], (i / kMgStages) & 1u, abort_flag) ||
          !mbar_wait(&acc_full[b], (i >> 1) & 1u, abort_flag)) {
        if (!*abort_flag) record_error(args.err, abort_flag, kErrTimeoutEpilogue);
        break;
      }
      tc_fence_after();
      uint32_t words[8];
      {
        const uint8_t* crow_s = c_s + s * kMgCBytes + crow * 64;
        const uint4 q0 = *reinterpret_cast<const uint4*>(crow_s + (((g0) ^ ((crow >> 1) & 3)) << 4));
        const uint4 q1 = *reinterpret_cast<const uint4*>(crow_s + (((g0 + 1) ^ ((crow >> 1) & 3)) << 4));
        words[0] = q0.x; words[1] = q0.y; words[2] = q0.z; words[3] = q0.w;
        words[4] = q1.x; words[5] = q1.y; words[6] = q1.z; words[7] = q1.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);  // this warp's codes are in registers
      if (kb_cur < args.K) {  // warp-uniform
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // 32-column chunks of the block
          uint32_t v[32];
          tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + b * kMgCols +
                                 col0 + h * 32,
                             v);
          tmem_ld_wait();
          if (h == 1) {  // this warp's part of buffer b is in registers
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[b]);
          }
          // stage row = this lane's row n, its 16-byte group w at slot w ^ ((lane >> 1) & 3)
          uint8_t* stage = stage1;
          if (chunks >= 1 && lane == 0) bulk_wait_group_read<0>();  // the previous store read it
          __syncwarp();
          ++chunks;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            uint32_t o[4], y[4];
            lut_decode8(words[4 * h + w], lut, o);  // elements 8w .. 8w+7 of the chunk
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              const float w_lo = __uint_as_float(o[p] << 16);
              const float w_hi = __uint_as_float(o[p] & 0xFFFF0000u);
              const int e = 8 * w + 2 * p;
              y[p] = pack_bf16x2_rn(__fmaf_rn(args.scale, __uint_as_float(v[e]), w_lo),
                                    __fmaf_rn(args.scale, __uint_as_float(v[e + 1]), w_hi));
            }
            *reinterpret_cast<uint4*>(stage + lane * 64 + ((w ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(y[0], y[1], y[2], y[3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0)  // rows past N are not written
            tma_store_2d(&tm_out, stage, static_cast<int>(kb_cur + h * 32),
                         static_cast<int>(n_cur - lane));
          if (lane == 0) bulk_commit_group();
        }
      } else {  // block past K: nothing to read, release the buffer
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[b]);
      }
    }
    if (lane == 0) bulk_wait_group_all();  // tile stores done before the CTA exits
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * kMgCols);
  }
}

}  // namespace

cudaError_t launch_merge_lora(const qlora_nf4_weight& w, const uint16_t* A, const uint16_t* B,
                              int r, float scale, uint16_t* out, cudaStream_t st) {
  MergeArgs a;
  a.c2 = w.c2;
  a.c1 = w.c1;
  a.mean = w.mean;
  a.N = w.n_out;
  a.K = w.k_in;
  a.r = r;
  a.scale = scale;
  a.out = out;
  a.row_tiles = static_cast<int>((w.n_out + kMgRows - 1) / kMgRows);
  a.num_tiles = a.row_tiles * static_cast<int>((w.k_in + kMgCols - 1) / kMgCols);
  a.err = device_error_word();
  CUtensorMap ta, tb, tc, to;
  // A [K, r]: rows k, 64-wide j box (zero past r); B [r, N]: 64 x 64 boxes of (n, j)
  if (!make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, r, w.k_in, static_cast<uint64_t>(r) * 2,
                    64, kMgCols, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, w.n_out, r, w.n_out * 2, 64, 64,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      // codes [N, K/2] bytes: 64-byte x 128-row boxes, 64-byte swizzle
      !make_tmap_2d(&tc, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.codes, w.k_in / 2, w.n_out, w.k_in / 2,
                    kMgCols / 2, kMgRows, CU_TENSOR_MAP_SWIZZLE_64B) ||
      // out [N, K]: 32 x 32 boxes (k inner), 64-byte swizzle
      !make_tmap_2d(&to, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, out, w.k_in, w.n_out, w.k_in * 2, 32, 32,
                    CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  auto kern = w.codebook == 1 ? k_merge_lora<1> : k_merge_lora<0>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMgSmem);
  if (e != cudaSuccess) return e;
  const int slots = num_sms() * kMgCtasPerSm;
  const int grid = a.num_tiles < slots ? a.num_tiles : slots;  // persistent
  if (grid == 0) return cudaSuccess;
  note_launches(1);
  kern<<<grid, kMgThreads, kMgSmem, st>>>(ta, tb, tc, to, a);
  return cudaGetLastError();
}

}  // namespace qlora
