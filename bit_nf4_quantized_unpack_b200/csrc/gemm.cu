// gemm.cu -- the QLoRA linear layer on the 5th-generation tensor cores (tcgen05, TMEM
// accumulators, TMA-fed shared memory) for M > 16 tokens.
//
// Forward (page "QLoRA", itwiki.kr, section "계산 방식"; alpha/r from page
// "quantization", minnong511 blog):  Y = X W_hat^T + scale (X A) B
// Backward (same sections): G = dY B^T, dX = dY W_hat + scale G A^T,
//                           dA = scale X^T G, dB = scale T^T dY.
//
// Kernels
//  k_fused_nf4_gemm<kForward>: D[n, m] = sum_k W_hat[n, k] X[m, k] + sum_j B[j, n] Ts[m, j]
//      W_hat is never written to memory: packed codes arrive by TMA, eight dequant
//      warps expand them (double dequantization, bit-exact bf16) straight into the
//      128B-swizzled shared-memory operand layout, and one thread issues
//      tcgen05.mma into a 128 x 256 fp32 TMEM accumulator. The LoRA product is two
//      more pipeline steps on the same accumulator with operands B (r padded to a
//      multiple of 16 with zeros by TMA) and Ts = scale T split into a bf16 hi part
//      and a bf16 lo part (scale T - hi), which keeps it at fp32-level accuracy.
//  k_fused_nf4_gemm<kDgrad>: D[k, m] = sum_n W_hat[n, k] dY[m, n] + sum_j A[k, j] Gs[m, j]
//      the same pipeline with W_hat dequantized into the MN-major operand layout
//      (contraction over the output features n).
//  k_lora_gemm: the rank-r products T = X A, G = dY B^T (split over the contraction)
//      and dA, dB (contraction over tokens; G and T enter as bf16 hi + lo pairs so
//      that the gradients keep fp32-level accuracy).
// Small elementwise kernels finalize the split partial sums.
#include <cuda_bf16.h>

#include <algorithm>
#include <utility>

#include "internal.h"
#include "nf4_device.cuh"

namespace qlora {
namespace {

// ================================================================== fused NF4 GEMM
enum class Mode { kForward, kDgrad };

// Warp roles of the persistent fused kernel:
//   warp 0      TMA producer of the token-side operand (and the LoRA operands)
//   warp 1      MMA issuer (one thread), owner of the TMEM allocation
//   warps 2-5   epilogue: TMEM -> registers -> bf16 -> shared -> TMA store, one TMEM lane
//               quarter each
//   warps 6-15  dequantization, two groups of four warps taking code steps in turn;
//               warps 9 and 13 stay idle so that no dequantizing warp shares the MMA
//               warp's scheduler (warp w issues from sub-partition w % 4): the single
//               MMA thread then issues at full rate between its ALU-heavy neighbours.
// A tile is 128 weight-side rows x 512 tokens held as two 256-column fp32 accumulators
// (all 512 TMEM columns): every dequantized 128 x 64 weight tile feeds 8 MMAs.
//
// Code step c (the c-th 64-wide contraction step of this CTA) belongs to warpgroup
// c % kDeqGroups and is dequantized into weight slot c % kWSlots; every slot therefore
// has one owner that uses it in order, so no mbarrier parity wait is ever more than one
// phase ahead. The owner loads the packed codes and block constants of its next step
// into registers and expands a step completely in registers before it waits for its
// slot to be free: only the shared-memory stores remain on the path between the MMAs
// of step c - kWSlots completing and step c being issued.
constexpr int kDeqGroups = 2;
constexpr int kWPerGroup = 2;
constexpr int kWSlots = kDeqGroups * kWPerGroup;
constexpr int kEpiWarp0 = 2;
constexpr int kDeqWarp0 = 6;
constexpr int kFusedThreads = 512;
static_assert(kDeqGroups == 2, "dequant warp map below has eight entries");
// position of a dequantizing warp in its groups (-1: not a dequantizing warp)
__device__ __forceinline__ int deq_index(int warp) {
  // warps 6 7 8 | 10 11 12 | 14 15  ->  0..7 ; 9, 13 (sub-partition 1) idle
  if (warp < kDeqWarp0 || warp == 9 || warp == 13) return -1;
  return warp - kDeqWarp0 - (warp > 9) - (warp > 13);
}
constexpr int kTileRows = 128;   // D rows on the weight side (n forward, k dgrad) = TMEM lanes
constexpr int kHalfCols = 256;   // tokens per MMA / per accumulator
constexpr int kHalves = 2;       // accumulators per tile
constexpr int kTileCols = kHalfCols * kHalves;  // tokens per tile
constexpr int kBK = 64;          // contraction per pipeline step
constexpr int kHalfSlots = 4;    // 256-token operand tiles in the ring
constexpr int kXSlots = kHalfSlots / 2;  // ring slots: the two half tiles of one step
constexpr uint32_t kHalfBytes = kHalfCols * kBK * 2;  // 32 KB
constexpr uint32_t kWBytes = kTileRows * kBK * 2;     // 16 KB
constexpr uint32_t kEpiBytes = 4 * 2 * 32 * 32 * 2;    // per epilogue warp: 2 x (32 tokens x 32 rows)
constexpr uint32_t kFusedSmem = kHalfSlots * kHalfBytes + (kWSlots + 1) * kWBytes + kEpiBytes +
                                1024 + 512 + 1024;
static_assert(kFusedSmem <= 227 * 1024, "shared memory per CTA");

struct FusedArgs {
  const uint8_t* codes;  // [N][K/2] packed NF4 codes (16-byte aligned)
  const uint8_t* c2;
  const float* c1;
  const float* mean;
  int64_t N, K, M;    // W is N x K, M tokens
  int ext_mmas;       // 16-wide MMAs per LoRA step (0: no LoRA steps)
  int row_tiles;      // tiles along the D rows (weight side)
  int num_tiles;      // row_tiles x token tiles
  uint16_t* out;      // [M, out_ld] bf16
  bool out_f32;       // write fp32 [M, out_ld] through tm_out instead (dgrad partial sums)
  int64_t out_ld;     // N (forward) or K (dgrad)
  int64_t out_rows;   // valid D rows: N (forward) or K (dgrad)
  int codebook;       // 4-bit codebook of the codes (0 NF4, 1 uniform)
  int* err;
};

template <Mode MODE, int CB>
__global__ void __launch_bounds__(kFusedThreads, 1)
    k_fused_nf4_gemm(const __grid_constant__ CUtensorMap tm_act,
                     const __grid_constant__ CUtensorMap tm_ext_w,
                     const __grid_constant__ CUtensorMap tm_ext_act,
                     const __grid_constant__ CUtensorMap tm_out, const FusedArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* act_s = smem;                             // [kXSlots][2][kHalfBytes] token side
  uint8_t* w_s = act_s + kHalfSlots * kHalfBytes;    // [kWSlots][kWBytes] dequantized
  uint8_t* wext_s = w_s + kWSlots * kWBytes;         // [kWBytes] LoRA weight-side operand
  uint16_t* epi_s = reinterpret_cast<uint16_t*>(wext_s + kWBytes);  // [4][2][32][32] staging
  uint64_t* bars = reinterpret_cast<uint64_t*>(wext_s + kWBytes + kEpiBytes);
  uint64_t* half_full = bars;                       // [kHalfSlots] a token tile landed
  uint64_t* x_empty = half_full + kHalfSlots;       // [kXSlots] MMAs reading a step's tiles done
  uint64_t* deq_full = x_empty + kXSlots;           // [kWSlots] dequantized tile ready
  uint64_t* w_empty = deq_full + kWSlots;           // [kWSlots] MMAs reading it done
  uint64_t* ext_empty = w_empty + kWSlots;          // LoRA operand slot read out
  uint64_t* acc_full = ext_empty + 1;               // [kHalves] accumulator complete
  uint64_t* acc_empty = acc_full + kHalves;         // [kHalves] accumulator read out
  uint64_t* mma_drain = acc_empty + kHalves;        // all MMAs of the CTA completed (exit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* t8 = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 512);  // [256]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x < 256) t8[threadIdx.x] = t8_value(threadIdx.x);
  const int64_t contraction = (MODE == Mode::kForward) ? args.K : args.N;
  const int ksteps = static_cast<int>((contraction + kBK - 1) / kBK);
  // the LoRA product enters as two steps: bf16 hi part, then bf16 lo part of scale*T
  const bool has_ext = args.ext_mmas > 0;
  const int total = ksteps + (has_ext ? 2 : 0);
  const int my_tiles = (static_cast<int>(blockIdx.x) < args.num_tiles)
                           ? (args.num_tiles - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1
                           : 0;
  // a tile whose second 256 tokens lie past M runs one accumulator only
  auto halves_in = [&](int64_t m0) { return (args.M - m0 > kHalfCols) ? kHalves : 1; };
  auto tile_coords = [&](int i, int64_t& row0, int64_t& m0) {
    const int tile = blockIdx.x + i * gridDim.x;
    row0 = static_cast<int64_t>(tile % args.row_tiles) * kTileRows;
    m0 = static_cast<int64_t>(tile / args.row_tiles) * kTileCols;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kHalfSlots; ++s) mbar_init(&half_full[s], 1);
    for (int s = 0; s < kXSlots; ++s) mbar_init(&x_empty[s], 1);
    for (int s = 0; s < kWSlots; ++s) {
      mbar_init(&deq_full[s], 4);
      mbar_init(&w_empty[s], 1);
    }
    mbar_init(ext_empty, 1);
    for (int h = 0; h < kHalves; ++h) {
      mbar_init(&acc_full[h], 1);
      mbar_init(&acc_empty[h], 4);
    }
    mbar_init(mma_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTileCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait_and_release();  // inputs of the previous kernel are complete from here on

  if (warp == 0) {
    // ------------------------------------------------ TMA: token-side operand, LoRA steps
    if (lane == 0) {
      tma_prefetch_desc(&tm_act);
      // step g fills slot g % kXSlots: half tile h in buffer 2 (g % kXSlots) + h, counted
      // on that buffer's own barrier (a tile with one accumulator leaves buffer 1 unused)
      int issued = 0;                  // steps; buffer 2 xs is loaded at every use of slot xs
      int h1_uses0 = 0, h1_uses1 = 0;  // loads of buffer 1 and buffer 3 (second halves)
      bool ok = true;
      for (int i = 0; i < my_tiles && ok; ++i) {
        int64_t row0, m0;
        tile_coords(i, row0, m0);
        const int nh = halves_in(m0);
        for (int step = 0; step < total && ok; ++step) {
          const bool ext = step >= ksteps;
          const bool ext_w = ext && step == ksteps;  // this step also brings the LoRA operand
          if (ext_w && i >= 1 && !mbar_wait(ext_empty, (i - 1) & 1u, abort_flag)) {
            record_error(args.err, abort_flag, kErrTimeoutProducer);
            ok = false;
            break;
          }
          const int xs = issued % kXSlots;
          if (issued >= kXSlots &&
              !mbar_wait(&x_empty[xs], ((issued / kXSlots) - 1) & 1u, abort_flag)) {
            record_error(args.err, abort_flag, kErrTimeoutProducer);
            ok = false;
            break;
          }
          for (int h = 0; h < nh; ++h) {
            const int hs = 2 * xs + h;
            const int mh = static_cast<int>(m0) + h * kHalfCols;
            if (h == 1) {
              if (xs == 0) ++h1_uses0;
              else ++h1_uses1;
            }
            if (!ext) {
              mbar_arrive_expect_tx(&half_full[hs], kHalfBytes);
              tma_load_2d(act_s + hs * kHalfBytes, &tm_act, &half_full[hs], step * kBK, mh);
            } else {
              const bool with_w = ext_w && h == 0;
              mbar_arrive_expect_tx(&half_full[hs], kHalfBytes + (with_w ? kWBytes : 0u));
              if (with_w) {
                if (MODE == Mode::kForward) {
                  // B [r, N] as an MN-major operand: two 64-wide chunks of n, rows j >= r are 0
                  tma_load_2d(wext_s, &tm_ext_w, &half_full[hs], static_cast<int>(row0), 0);
                  tma_load_2d(wext_s + 8192, &tm_ext_w, &half_full[hs], static_cast<int>(row0) + 64,
                              0);
                } else {
                  // A [K, r] as a K-major operand (columns j >= r are 0)
                  tma_load_2d(wext_s, &tm_ext_w, &half_full[hs], 0, static_cast<int>(row0));
                }
              }
              tma_load_2d(act_s + hs * kHalfBytes, &tm_ext_act, &half_full[hs],
                          (step - ksteps) * 64, mh);
            }
          }
          ++issued;
        }
      }
      if (*abort_flag) {  // let copies already in flight land before the CTA exits
        for (int xs = 0; xs < kXSlots; ++xs) {
          const int u0 = issued / kXSlots + (xs < issued % kXSlots ? 1 : 0);  // buffer 2 xs
          const int u1 = xs == 0 ? h1_uses0 : h1_uses1;                       // buffer 2 xs + 1
          if (u0 > 0) mbar_wait_drain(&half_full[2 * xs], (u0 - 1) & 1u);
          if (u1 > 0) mbar_wait_drain(&half_full[2 * xs + 1], (u1 - 1) & 1u);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_main =
          idesc_bf16_f32(kTileRows, kHalfCols, MODE == Mode::kDgrad, false);
      constexpr uint32_t idesc_ext =
          idesc_bf16_f32(kTileRows, kHalfCols, MODE == Mode::kForward, false);
      // Descriptor deltas per 16-wide K slice (start address field counts 16-byte units):
      // K-major operands advance 32 bytes; the MN-major dequantized dgrad tile advances
      // two 8-row groups (4096 bytes); the MN-major LoRA operand B [r, N] one 16-row
      // slice of its 64-row chunk (2048 bytes).
      constexpr uint32_t kDA = (MODE == Mode::kForward) ? 2u : 256u;
      constexpr uint32_t kDX = (MODE == Mode::kForward) ? 128u : 2u;
      const uint64_t desc_ext = (MODE == Mode::kForward)
                                    ? smem_desc_sw128(smem_u32(wext_s), 8192, 1024)
                                    : smem_desc_sw128(smem_u32(wext_s), 16, 1024);
      bool ok = true;
      int steps_done = 0, main_done = 0, ext_done = 0;
      int h1_uses0 = 0, h1_uses1 = 0;  // loads consumed from buffers 1 and 3 (second halves)
      int acc_uses[kHalves] = {0, 0};  // tiles accumulated so far in each accumulator
      for (int i = 0; i < my_tiles && ok; ++i) {
        int64_t row0, m0;
        tile_coords(i, row0, m0);
        const int nh = halves_in(m0);
        for (int step = 0; step < total && ok; ++step) {
          const bool main_step = step < ksteps;
          const int c = i * ksteps + step;  // code step of a main step
          uint64_t da;
          if (main_step) {
            const int ws = c % kWSlots;
            if (!mbar_wait(&deq_full[ws], (c / kWSlots) & 1u, abort_flag)) {
              record_error(args.err, abort_flag, kErrTimeoutMma);
              ok = false;
              break;
            }
            da = (MODE == Mode::kForward) ? smem_desc_sw128(smem_u32(w_s + ws * kWBytes), 16, 1024)
                                          : smem_desc_sw128(smem_u32(w_s + ws * kWBytes), 1024, 2048);
          } else {
            da = desc_ext;  // landed with the first half tile of the first LoRA step
          }
          const int xs = steps_done % kXSlots;
          for (int h = 0; h < nh; ++h) {
            const int hs = 2 * xs + h;
            // the epilogue has read accumulator h of the previous tile out
            if (step == 0 && acc_uses[h] >= 1) {
              if (!mbar_wait(&acc_empty[h], (acc_uses[h] - 1) & 1u, abort_flag)) {
                record_error(args.err, abort_flag, kErrTimeoutMma);
                ok = false;
                break;
              }
              tc_fence_after();
            }
            // buffer 2 xs is loaded at every use of slot xs; buffer 2 xs + 1 only when the
            // tile has a second half
            const int uses = h == 0 ? steps_done / kXSlots : (xs == 0 ? h1_uses0 : h1_uses1);
            if (!mbar_wait(&half_full[hs], uses & 1u, abort_flag)) {
              record_error(args.err, abort_flag, kErrTimeoutMma);
              ok = false;
              break;
            }
            if (h == 1) {
              if (xs == 0) ++h1_uses0;
              else ++h1_uses1;
            }
            const uint32_t tmem_d = tmem_base + h * kHalfCols;
            const uint64_t db = smem_desc_sw128(smem_u32(act_s + hs * kHalfBytes), 16, 1024);
            if (main_step) {
              umma_bf16(tmem_d, da, db, idesc_main, step != 0);
#pragma unroll
              for (int kk = 1; kk < kBK / 16; ++kk)
                umma_bf16(tmem_d, da + kk * kDA, db + kk * 2u, idesc_main, 1u);
            } else {
              for (int kk = 0; kk < args.ext_mmas; ++kk)
                umma_bf16(tmem_d, da + kk * kDX, db + kk * 2u, idesc_ext, 1u);
            }
            if (step == total - 1) {  // accumulator h of this tile is complete
              umma_commit(&acc_full[h]);
              ++acc_uses[h];
            }
          }
          if (!ok) break;
          umma_commit(&x_empty[xs]);  // the step's token tiles are read
          ++steps_done;
          if (main_step) {
            umma_commit(&w_empty[c % kWSlots]);
            ++main_done;
          } else if (step == total - 1) {
            umma_commit(ext_empty);
            ++ext_done;
          }
        }
      }
      // every MMA this thread issued has completed before TMEM is freed (on the normal
      // path and after an abort alike); the barrier is used for this one phase only
      umma_commit(mma_drain);
      mbar_wait_drain(mma_drain, 0);
      // the commits of the last steps arrive asynchronously on barriers nobody else waits
      // for any more: let them land before the CTA (and its shared memory) goes
      uint32_t par;
      for (int s = 0; s < kXSlots; ++s)
        if (last_use(steps_done, kXSlots, s, par)) mbar_wait_drain(&x_empty[s], par);
      for (int s = 0; s < kWSlots; ++s)
        if (last_use(main_done, kWSlots, s, par)) mbar_wait_drain(&w_empty[s], par);
      if (last_use(ext_done, 1, 0, par)) mbar_wait_drain(ext_empty, par);
      for (int h = 0; h < kHalves; ++h)
        if (acc_uses[h] >= 1) mbar_wait_drain(&acc_full[h], (acc_uses[h] - 1) & 1u);
    }
  } else if (deq_index(warp) >= 0) {
    // ------------------------------------------------ dequantization
    const int dw = deq_index(warp);
    const int wg = dw >> 2;                  // warpgroup: code steps wg, wg + kDeqGroups, ...
    const int local = (dw & 3) * 32 + lane;  // 0..127
    const float mean = *args.mean;
    const int64_t bpr = args.K / 64;     // 64-blocks per weight row
    const int64_t code_ld = args.K / 2;  // bytes per weight row of codes
    const int ncodes = my_tiles * ksteps;
    // Code step c = tile i * ksteps + step t; this warpgroup walks c = wg, wg + kDeqGroups,
    // ... (i, t) and the tile origin are advanced incrementally (no divisions per step).
    struct Cursor {
      int i, t;
      int64_t row0, m0;
    };
    auto advance = [&](Cursor& k, int by) {
      k.t += by;
      while (k.t >= ksteps) {
        k.t -= ksteps;
        ++k.i;
      }
    };
    auto set_tile = [&](Cursor& k) { tile_coords(k.i, k.row0, k.m0); };
    // This thread's 64-block at a cursor: weight row n, block kb along K. Forward: one
    // block per D row; dgrad: two threads per contraction row n, 64 D rows (k) each.
    // Loads its 32 code bytes and block constants; false outside W.
    auto fetch = [&](const Cursor& k, uint4& a, uint4& b, uint32_t& e2, float& e1) {
      int64_t n, kb;
      if (MODE == Mode::kForward) {
        n = k.row0 + local;
        kb = k.t;
      } else {
        n = static_cast<int64_t>(k.t) * kBK + (local >> 1);
        kb = k.row0 / 64 + (local & 1);
      }
      if (n >= args.N || kb >= bpr) return false;
      const uint4* src = reinterpret_cast<const uint4*>(args.codes + n * code_ld + kb * 32);
      a = __ldg(src);
      b = __ldg(src + 1);
      const int64_t j = n * bpr + kb;
      e2 = __ldg(args.c2 + j);
      e1 = __ldg(args.c1 + (j >> 8));
      return true;
    };
    Cursor cur{0, 0, 0, 0};
    advance(cur, wg);
    set_tile(cur);
    uint4 qa = make_uint4(0u, 0u, 0u, 0u), qb = qa;  // the next step's codes
    uint32_t e2n = 0u;
    float e1n = 0.f;
    bool vn = (wg < ncodes) && fetch(cur, qa, qb, e2n, e1n);
    Cursor nxt = cur;
    advance(nxt, kDeqGroups);
    if (nxt.i < my_tiles) set_tile(nxt);
    for (int c = wg; c < ncodes; c += kDeqGroups) {
      const uint32_t words[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
      const float sc = vn ? block_scale_tab(t8, e2n, e1n, mean) : 0.f;  // zeros outside W
      if (c + kDeqGroups < ncodes) vn = fetch(nxt, qa, qb, e2n, e1n);
      cur = nxt;
      advance(nxt, kDeqGroups);
      if (nxt.i != cur.i && nxt.i < my_tiles) set_tile(nxt);
      Nf4Lut lut;
      build_lut<CB>(sc, lut);
      uint32_t o[8][4];
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) lut_decode8(words[ch], lut, o[ch]);
      const int ws = c % kWSlots;
      if (c >= kWSlots && !mbar_wait(&w_empty[ws], ((c / kWSlots) - 1) & 1u, abort_flag)) {
        record_error(args.err, abort_flag, kErrTimeoutDequant);
        break;
      }
      uint8_t* dst = w_s + ws * kWBytes;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        uint32_t off;
        if (MODE == Mode::kForward) {
          off = sw128_kmajor_offset(local, ch);
        } else {
          const uint32_t nr = local >> 1;  // K-row (contraction) index inside the tile
          off = (nr >> 3) * 2048u + (local & 1) * 1024u + (nr & 7u) * 128u +
                ((ch ^ (nr & 7u)) << 4);
        }
        *reinterpret_cast<uint4*>(dst + off) = make_uint4(o[ch][0], o[ch][1], o[ch][2], o[ch][3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&deq_full[ws]);
    }
  } else if (warp >= kEpiWarp0 && warp < kDeqWarp0) {
    // ------------------------------------------------ epilogue
    // TMEM lane = D row, column = token. Each 32 x 32 chunk is transposed through shared
    // memory (stage[token][row]) into the token-major output's layout.
    const int quarter = warp & 3;  // TMEM lanes this warp may read
    uint16_t* stage2 = epi_s + quarter * (2 * 32 * 32);  // two stage buffers, used in turn
    int chunks = 0;                                      // chunks staged by this warp
    if (lane == 0) tma_prefetch_desc(&tm_out);
    int uses[kHalves] = {0, 0};
    bool ok = true;
    for (int i = 0; i < my_tiles && ok; ++i) {
      int64_t row0, m0;
      tile_coords(i, row0, m0);
      const int nh = halves_in(m0);
      const int64_t obase = row0 + quarter * 32;  // first D row of this warp
      for (int h = 0; h < nh; ++h) {
        if (!mbar_wait(&acc_full[h], uses[h] & 1u, abort_flag)) {
          if (!*abort_flag) record_error(args.err, abort_flag, kErrTimeoutEpilogue);
          ok = false;
          break;
        }
        ++uses[h];
        tc_fence_after();
        const uint32_t taddr =
            tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + h * kHalfCols;
        // One 32-token chunk: two 16-lane TMEM loads in the accumulator-fragment layout,
        // bf16 pairs, four transposing stmatrix into stage[token][row], then one TMA tile
        // store. A token's 64-byte stage row holds four 16-byte row groups, group g at
        // slot g ^ ((token >> 1) & 3), so the eight rows of each stored matrix fall in
        // distinct banks. The warp's two stage buffers alternate between chunks.
        auto slot_of = [](int tok, int g) { return static_cast<uint32_t>(tok * 64 + ((g ^ ((tok >> 1) & 3)) << 4)); };
        // chunks of this half inside M; the accumulator is released right after the last
        // one's TMEM load, before its conversion and store
        const int64_t left = (args.M - m0 - h * kHalfCols + 31) / 32;
        const int nchunks = left < kHalfCols / 32 ? static_cast<int>(left) : kHalfCols / 32;
        if (args.out_f32) {
          // fp32 output: one 32 x 32 chunk fills the warp's whole 4 KB stage, as
          // stage[token][row] (a 32-lane store per token is one 128-byte row), then one
          // unswizzled TMA tile store; the stage is reused once that store has read it
#pragma unroll 1
          for (int c = 0; c < nchunks; ++c) {
            const int64_t mb = m0 + h * kHalfCols + c * 32;
            const uint32_t stage_s = smem_u32(stage2);
            if (chunks >= 1 && lane == 0) bulk_wait_group_read<0>();
            __syncwarp();
            ++chunks;
            uint32_t v[32];
            tmem_ld_32x32b_x32(taddr + c * 32, v);  // row quarter * 32 + lane, 32 tokens
            tmem_ld_wait();
            if (c == nchunks - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&acc_empty[h]);
            }
#pragma unroll
            for (int j = 0; j < 32; ++j)
              asm volatile("st.shared.b32 [%0], %1;" ::"r"(stage_s + j * 128 + lane * 4), "r"(v[j])
                           : "memory");
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && obase < args.out_rows) {
              tma_store_2d(&tm_out, stage2, static_cast<int>(obase), static_cast<int>(mb));
              bulk_commit_group();
            }
          }
          continue;
        }
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
          const int64_t mb = m0 + h * kHalfCols + c * 32;
          uint16_t* stage = stage2 + (chunks & 1) * (32 * 32);
          const uint32_t stage_s = smem_u32(stage);
          // the tile store issued from this buffer two chunks ago has read it
          if (chunks >= 2 && lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
          ++chunks;
          uint32_t a[16], b[16];
          tmem_ld_16x256b_x4(taddr + c * 32, a);                 // rows 0-15 of the quarter
          tmem_ld_16x256b_x4(taddr + (16u << 16) + c * 32, b);   // rows 16-31
          tmem_ld_wait();
          if (c == nchunks - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[h]);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {  // tokens 8j..8j+7 of the chunk
            // matrix m = row group m (8 rows), its stored row i = token 8j + i
            const int tok = 8 * j + (lane & 7);
            stmatrix_x4_trans(stage_s + slot_of(tok, lane >> 3),
                              pack_bf16x2_rn(__uint_as_float(a[4 * j]), __uint_as_float(a[4 * j + 1])),
                              pack_bf16x2_rn(__uint_as_float(a[4 * j + 2]), __uint_as_float(a[4 * j + 3])),
                              pack_bf16x2_rn(__uint_as_float(b[4 * j]), __uint_as_float(b[4 * j + 1])),
                              pack_bf16x2_rn(__uint_as_float(b[4 * j + 2]), __uint_as_float(b[4 * j + 3])));
          }
          // the stage's 64-byte rows and their 16-byte group swizzle are the tensor map's
          // box (32 rows x 32 tokens) and its 64-byte swizzle; rows and tokens outside
          // the output are not written
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && obase < args.out_rows) {
            tma_store_2d(&tm_out, stage, static_cast<int>(obase), static_cast<int>(mb));
            bulk_commit_group();
          }
        }
      }
    }
    if (lane == 0) bulk_wait_group_all();  // tile stores done before the CTA exits
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTileCols);
  }
}

// ================================================================== LoRA GEMMs
constexpr int kLoraThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr uint32_t kLoraABytes = 128 * kBK * 2;  // 16 KB
// Pipeline depth: shared memory stays under 113 KB so that two CTAs share an SM.
__host__ __device__ constexpr int lora_stages(int nc) { return nc == 128 ? 3 : 4; }
__host__ __device__ constexpr uint32_t lora_smem(int nc) {
  return lora_stages(nc) * (kLoraABytes + nc * kBK * 2) + 1024 + 256;
}
constexpr int kLoraCtasPerSm = 2;
static_assert(lora_smem(128) <= 113 * 1024 && lora_smem(64) <= 113 * 1024, "two CTAs per SM");

struct LoraArgs {
  int steps_total;   // 64-wide contraction steps
  int steps_per;     // steps per split
  int tiles0;        // row tiles of the first problem; later tiles belong to the second
  float* partial;    // [splits][rows_pad][64] fp32 (NC = 128: hi + lo columns summed)
  int64_t rows_pad;  // the problems' row tiles stacked: 128 x (tiles0 + tiles of the second)
  int* err;
};

// D[128-row tile, NC] = sum over this CTA's contraction range of A^T B (both bf16,
// K-major or MN-major 128B-swizzled tiles loaded by TMA). With NC = 128 the B operand is
// a bf16 hi | lo pair and the partial written is D[:, j] + D[:, 64 + j].
// One launch may run two problems with the same contraction (operands tm_a/tm_b for
// the first tiles0 row tiles, tm_a1/tm_b1 after); their partial rows are stacked.
template <bool A_MN, bool B_MN, int NC>
__global__ void __launch_bounds__(kLoraThreads, 1)
    k_lora_gemm(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_a1,
                const __grid_constant__ CUtensorMap tm_b1, const LoraArgs args) {
  constexpr uint32_t kB = NC * kBK * 2;
  constexpr int kLoraStages = lora_stages(NC);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* a_s = smem;
  uint8_t* b_s = a_s + kLoraStages * kLoraABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(b_s + kLoraStages * kB);
  uint64_t* full = bars;
  uint64_t* empty = bars + kLoraStages;
  uint64_t* acc_full = bars + 2 * kLoraStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kLoraStages + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool second = static_cast<int>(blockIdx.x) >= args.tiles0;
  const CUtensorMap* map_a = second ? &tm_a1 : &tm_a;
  const CUtensorMap* map_b = second ? &tm_b1 : &tm_b;
  // row of the operand (TMA coordinate) and of the stacked partial
  const int64_t row0 = static_cast<int64_t>(second ? blockIdx.x - args.tiles0 : blockIdx.x) * 128;
  const int64_t prow0 = static_cast<int64_t>(blockIdx.x) * 128;
  const int s_begin = blockIdx.y * args.steps_per;
  const int s_end = std::min(args.steps_total, s_begin + args.steps_per);
  const int nsteps = std::max(0, s_end - s_begin);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kLoraStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, NC);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  griddep_wait_and_release();

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % kLoraStages;
        const uint32_t use = i / kLoraStages;
        if (i >= kLoraStages && !mbar_wait(&empty[s], (use - 1) & 1u, abort_flag)) {
          record_error(args.err, abort_flag, kErrTimeoutProducer);
          break;
        }
        const int kc = (s_begin + i) * kBK;  // contraction coordinate
        mbar_arrive_expect_tx(&full[s], kLoraABytes + kB);
        if (A_MN) {
          tma_load_2d(a_s + s * kLoraABytes, map_a, &full[s], static_cast<int>(row0), kc);
          tma_load_2d(a_s + s * kLoraABytes + 8192, map_a, &full[s], static_cast<int>(row0) + 64,
                      kc);
        } else {
          tma_load_2d(a_s + s * kLoraABytes, map_a, &full[s], kc, static_cast<int>(row0));
        }
        if (B_MN) {
#pragma unroll
          for (int c = 0; c < NC / 64; ++c)
            tma_load_2d(b_s + s * kB + c * 8192, map_b, &full[s], c * 64, kc);
        } else {
          tma_load_2d(b_s + s * kB, map_b, &full[s], kc, 0);
        }
        ++issued;
      }
      if (*abort_flag)
        for (int i = std::max(0, issued - kLoraStages); i < issued; ++i)
          mbar_wait_drain(&full[i % kLoraStages], (i / kLoraStages) & 1u);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, NC, A_MN, B_MN);
      bool ok = true;
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % kLoraStages;
        if (!mbar_wait(&full[s], (i / kLoraStages) & 1u, abort_flag)) {
          record_error(args.err, abort_flag, kErrTimeoutMma);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(a_s + s * kLoraABytes);
        const uint32_t b0 = smem_u32(b_s + s * kB);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t ad = A_MN ? smem_desc_sw128(a0 + kk * 2048, 8192, 1024)
                                   : smem_desc_sw128(a0 + kk * 32, 16, 1024);
          const uint64_t bd = B_MN ? smem_desc_sw128(b0 + kk * 2048, 8192, 1024)
                                   : smem_desc_sw128(b0 + kk * 32, 16, 1024);
          umma_bf16(tmem_d, ad, bd, idesc, (i | kk) != 0);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(acc_full);
      if (!ok) mbar_wait_drain(acc_full, 0);
      // let the last commits arrive before the CTA's shared memory is released
      for (int s = 0; s < kLoraStages; ++s) {
        const int last = nsteps - 1 - ((nsteps - 1 - s) % kLoraStages + kLoraStages) % kLoraStages;
        if (ok && last >= 0 && last < nsteps) mbar_wait_drain(&empty[s], (last / kLoraStages) & 1u);
      }
      mbar_wait_drain(acc_full, 0);
    }
  } else {
    const bool have = nsteps > 0;
    if (!have || (mbar_wait(acc_full, 0, abort_flag) && !*abort_flag)) {
      tc_fence_after();
      const int quarter = warp & 3;
      const int64_t row = prow0 + quarter * 32 + lane;
      float* dst = args.partial + (static_cast<int64_t>(blockIdx.y) * args.rows_pad + row) * 64;
      const uint32_t taddr = tmem_d + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t v[32];
        if (have) {
          tmem_ld_32x32b_x32(taddr + c * 32, v);
          tmem_ld_wait();
          if (NC == 128) {  // add the lo half of the pair
            uint32_t w[32];
            tmem_ld_32x32b_x32(taddr + 64 + c * 32, w);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i)
              v[i] = __float_as_uint(__uint_as_float(v[i]) + __uint_as_float(w[i]));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0u;
        }
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<uint4*>(dst + c * 32 + i) = make_uint4(v[i], v[i + 1], v[i + 2], v[i + 3]);
      }
    } else if (!*abort_flag) {
      record_error(args.err, abort_flag, kErrTimeoutEpilogue);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, NC);
  }
}

// ================================================================== finalize kernels
// T (or G) = sum of split partials [S][rows_pad][64]. Writes, where asked:
//   plain fp32 [M, r]; bf16 hi/lo of scale * v [M, 128] (the K-extension operand);
//   bf16 hi/lo of v [M, 128] (operand of the LoRA gradients).
//   With t_in, also the bf16 hi/lo pair [M, 128] of that fp32 [M, r] (into t_hilo).
__global__ void k_finalize_rank(const float* __restrict__ part, int splits, int64_t rows_pad,
                                int64_t M, int r, float scale, float* __restrict__ plain,
                                uint16_t* __restrict__ scaled, uint16_t* __restrict__ hilo,
                                const float* __restrict__ t_in, uint16_t* __restrict__ t_hilo) {
  griddep_wait_and_release();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= M * 64) return;
  const int64_t m = i >> 6;
  const int j = static_cast<int>(i & 63);
  float v = 0.f;
  const float* p = part + m * 64 + j;
  const int64_t stride = rows_pad * 64;
  int sp = 0;
  float v1 = 0.f, v2 = 0.f, v3 = 0.f;
  for (; sp + 4 <= splits; sp += 4) {  // four independent loads in flight
    v += p[sp * stride];
    v1 += p[(sp + 1) * stride];
    v2 += p[(sp + 2) * stride];
    v3 += p[(sp + 3) * stride];
  }
  for (; sp < splits; ++sp) v += p[sp * stride];
  v = (v + v1) + (v2 + v3);
  if (j >= r) v = 0.f;
  if (plain && j < r) plain[m * r + j] = v;
  if (scaled) {  // [M, 128]: bf16 hi | bf16 lo of scale * v
    const float sv = v * scale;
    const uint16_t hi = bf16_bits_rn(sv);
    scaled[m * 128 + j] = hi;
    scaled[m * 128 + 64 + j] = bf16_bits_rn(sv - __uint_as_float(static_cast<uint32_t>(hi) << 16));
  }
  if (hilo) {
    const uint16_t hi = bf16_bits_rn(v);
    const float hv = __uint_as_float(static_cast<uint32_t>(hi) << 16);
    hilo[m * 128 + j] = hi;
    hilo[m * 128 + 64 + j] = bf16_bits_rn(v - hv);
  }
  if (t_hilo) {
    const float tv = (j < r) ? t_in[m * r + j] : 0.f;
    const uint16_t hi = bf16_bits_rn(tv);
    t_hilo[m * 128 + j] = hi;
    t_hilo[m * 128 + 64 + j] = bf16_bits_rn(tv - __uint_as_float(static_cast<uint32_t>(hi) << 16));
  }
}

// Both LoRA gradients from the stacked partials of one grouped launch:
//   rows [0, pad0) of P:  dA[k, j]   = scale * sum_s P[s][k][j]          ([rows0, r])
//   rows [pad0, ...):     dB[j, n]   = scale * sum_s P[s][pad0 + n][j]   ([r, rows1])
// One block per 16 stacked rows, four (row, j) items per thread with their split loads
// interleaved; a shared-memory tile gives coalesced writes in either orientation.
constexpr int kGradRows = 16;
static_assert(128 % kGradRows == 0, "a block of rows never straddles the two problems");
__global__ void __launch_bounds__(256)
    k_finalize_grad(const float* __restrict__ part, int splits, int64_t rows_pad, int64_t pad0,
                    int64_t rows0, float* __restrict__ out0, int64_t rows1,
                    float* __restrict__ out1, int r, float scale) {
  griddep_wait_and_release();
  __shared__ float tile[kGradRows][65];
  const int64_t srow0 = static_cast<int64_t>(blockIdx.x) * kGradRows;  // stacked
  const bool transpose = srow0 >= pad0;
  const int64_t row0 = transpose ? srow0 - pad0 : srow0;
  const int64_t rows = transpose ? rows1 : rows0;
  float* __restrict__ out = transpose ? out1 : out0;
  const int64_t stride = rows_pad * 64;
  float v[4] = {0.f, 0.f, 0.f, 0.f};
  const float* p = part + srow0 * 64 + threadIdx.x;  // item u: srow0 * 64 + threadIdx.x + 256 u
  for (int sp = 0; sp < splits; ++sp) {
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] += p[sp * stride + 256 * u];
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int idx = threadIdx.x + 256 * u;
    const int rl = idx >> 6, j = idx & 63;
    tile[rl][j] = (j < r && row0 + rl < rows) ? scale * v[u] : 0.f;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < kGradRows * r; idx += blockDim.x) {
    if (transpose) {  // out [r, rows]
      const int j = idx / kGradRows, rl = idx % kGradRows;
      if (row0 + rl < rows) out[static_cast<int64_t>(j) * rows + row0 + rl] = tile[rl][j];
    } else {          // out [rows, r]
      const int rl = idx / r, j = idx % r;
      if (row0 + rl < rows) out[(row0 + rl) * r + j] = tile[rl][j];
    }
  }
}

// ================================================================== host side
constexpr CUtensorMapDataType kBF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
constexpr CUtensorMapSwizzle kSW128 = CU_TENSOR_MAP_SWIZZLE_128B;

struct SplitPlan {
  int splits, steps_per, steps_total;
  int64_t tiles, rows_pad;
};

SplitPlan plan_split(int64_t rows, int64_t contraction) {
  SplitPlan p;
  p.tiles = (rows + 127) / 128;
  p.rows_pad = p.tiles * 128;
  p.steps_total = static_cast<int>((contraction + kBK - 1) / kBK);
  if (p.steps_total == 0 || p.tiles == 0) {  // empty operand: one (idle) split
    p.splits = 1;
    p.steps_per = p.steps_total > 0 ? p.steps_total : 1;
    return p;
  }
  // choose the split count that minimises (rounds of CTAs) x (steps per CTA + a fixed
  // per-CTA cost of about three steps)
  const int64_t slots = static_cast<int64_t>(kLoraCtasPerSm) * num_sms();
  int64_t best = -1;
  for (int want = 1; want <= p.steps_total && want <= 64; ++want) {
    const int per = (p.steps_total + want - 1) / want;
    const int splits = (p.steps_total + per - 1) / per;
    if (splits != want) continue;
    const int64_t rounds = (p.tiles * splits + slots - 1) / slots;
    const int64_t cost = rounds * (per + 3);
    if (best < 0 || cost < best) {
      best = cost;
      p.steps_per = per;
      p.splits = splits;
    }
  }
  return p;
}

// Largest partial buffer (floats) the plans of one call may need.
size_t partial_floats(int64_t rows, int64_t contraction, int nc) {
  const SplitPlan p = plan_split(rows, contraction);
  (void)nc;
  return static_cast<size_t>(p.splits) * p.rows_pad * 64;
}

// Launch on `st` with programmatic stream serialization: the kernel may begin (its
// prologue) while the stream's previous kernel drains; every kernel of this file waits
// for its predecessor with griddep_wait_and_release before it touches global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  note_launches(1);
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// G and T of a column-sharded backward (plain fp32 [M, r]; G summed over the shards) as
// the bf16 operand pairs of the fused dX kernel and the grouped dA/dB GEMM: scale G as
// hi | lo ([M, 128]), G as hi | lo and T as hi | lo (the arithmetic of k_finalize_rank).
__global__ void k_rank_from_plain(const float* __restrict__ G, const float* __restrict__ T,
                                  int64_t M, int r, float scale, uint16_t* __restrict__ gs,
                                  uint16_t* __restrict__ ghl, uint16_t* __restrict__ thl) {
  griddep_wait_and_release();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= M * 64) return;
  const int64_t m = i >> 6;
  const int j = static_cast<int>(i & 63);
  const float g = j < r ? G[m * r + j] : 0.f;
  const float t = j < r ? T[m * r + j] : 0.f;
  auto hilo = [&](uint16_t* out, float v) {
    const uint16_t hi = bf16_bits_rn(v);
    out[m * 128 + j] = hi;
    out[m * 128 + 64 + j] = bf16_bits_rn(v - __uint_as_float(static_cast<uint32_t>(hi) << 16));
  };
  hilo(gs, g * scale);
  hilo(ghl, g);
  hilo(thl, t);
}

// dst[i] = bf16_rn(src[i]), four per thread (n % 4 == 0, 16-byte aligned).
__global__ void k_to_bf16(const float4* __restrict__ src, uint2* __restrict__ dst, int64_t n4) {
  griddep_wait_and_release();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 v = src[i];
    dst[i] = make_uint2(pack_bf16x2_rn(v.x, v.y), pack_bf16x2_rn(v.z, v.w));
  }
}

// Stacked rows of a grouped launch: the first problem padded to whole tiles, then the second.
inline int64_t stacked_rows(int64_t rows0, int64_t rows1) { return align_up(rows0, 128) + rows1; }

// One problem (ta, tb over `rows`), or two with the same contraction when ta1/tb1 are given
// (rows0 = rows of the first, rows1 of the second; partial rows stacked).
template <bool A_MN, bool B_MN, int NC>
cudaError_t run_lora_gemm(const CUtensorMap& ta, const CUtensorMap& tb, int64_t rows0,
                          int64_t contraction, float* partial, cudaStream_t st, int* splits_out,
                          const CUtensorMap* ta1 = nullptr, const CUtensorMap* tb1 = nullptr,
                          int64_t rows1 = 0) {
  const int64_t rows = ta1 ? stacked_rows(rows0, rows1) : rows0;
  const SplitPlan p = plan_split(rows, contraction);
  LoraArgs a;
  a.tiles0 = ta1 ? static_cast<int>((rows0 + 127) / 128) : static_cast<int>(p.tiles);
  a.steps_total = p.steps_total;
  a.steps_per = p.steps_per;
  a.partial = partial;
  a.rows_pad = p.rows_pad;
  a.err = device_error_word();
  auto kern = k_lora_gemm<A_MN, B_MN, NC>;
  const uint32_t smem = lora_smem(NC);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  *splits_out = p.splits;
  return launch_pdl(kern, dim3(static_cast<unsigned>(p.tiles), static_cast<unsigned>(p.splits)),
                    dim3(kLoraThreads), smem, st, ta, tb, ta1 ? *ta1 : ta, tb1 ? *tb1 : tb, a);
}

template <Mode MODE>
cudaError_t run_fused(const CUtensorMap& ta, const CUtensorMap& tw, const CUtensorMap& tx,
                      const CUtensorMap& to, FusedArgs args, cudaStream_t st) {
  auto kern = args.codebook == 1 ? k_fused_nf4_gemm<MODE, 1> : k_fused_nf4_gemm<MODE, 0>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kFusedSmem);
  if (e != cudaSuccess) return e;
  const int64_t rows = (MODE == Mode::kForward) ? args.N : args.K;
  args.row_tiles = static_cast<int>((rows + kTileRows - 1) / kTileRows);
  args.num_tiles = args.row_tiles * static_cast<int>((args.M + kTileCols - 1) / kTileCols);
  const int grid = std::min(args.num_tiles, num_sms());  // persistent: one CTA per SM
  cudaEvent_t before, after;
  profile_events(&before, &after);
  if (before) {
    e = cudaEventRecord(before, st);
    if (e != cudaSuccess) return e;
  }
  e = launch_pdl(kern, dim3(grid), dim3(kFusedThreads), kFusedSmem, st, ta, tw, tx, to, args);
  if (e == cudaSuccess && after) e = cudaEventRecord(after, st);
  return e;
}

inline unsigned blocks_for(int64_t n, int t) { return static_cast<unsigned>((n + t - 1) / t); }

// Workspace carving: a bump allocator over the caller's buffer.
struct Carve {
  char* base;
  size_t off = 0;
  explicit Carve(void* b) : base(static_cast<char*>(b)) {}
  template <typename T>
  T* take(size_t count) {
    off = align_up(off, 256);
    T* p = reinterpret_cast<T*>(base ? base + off : nullptr);
    off += count * sizeof(T);
    return p;
  }
};

size_t fwd_layout(const LinearShape& s, void* ws, float** part, uint16_t** ts) {
  Carve c(ws);
  *part = c.take<float>(partial_floats(s.M, s.K, 64));
  *ts = c.take<uint16_t>(static_cast<size_t>(s.M) * 128);
  return c.off + 256;
}

size_t bwd_layout(const LinearShape& s, void* ws, float** part, uint16_t** gs, uint16_t** ghl,
                  uint16_t** thl, float** t) {
  Carve c(ws);
  size_t pf = partial_floats(s.M, s.N, 64);                    // G = dY B^T
  pf = std::max(pf, partial_floats(s.M, s.K, 64));             // T = X A (recompute)
  pf = std::max(pf, partial_floats(stacked_rows(s.K, s.N), s.M, 128));  // dA and dB
  *part = c.take<float>(pf);
  *gs = c.take<uint16_t>(static_cast<size_t>(s.M) * 128);
  *ghl = c.take<uint16_t>(static_cast<size_t>(s.M) * 128);
  *thl = c.take<uint16_t>(static_cast<size_t>(s.M) * 128);
  *t = c.take<float>(static_cast<size_t>(s.M) * s.r);
  return c.off + 256;
}

#define QL_TRY(expr)                                  \
  do {                                                \
    cudaError_t _e = (expr);                          \
    if (_e != cudaSuccess) return cuda_status(_e);    \
  } while (0)
#define QL_MAP(...)                                                    \
  do {                                                                 \
    if (!make_tmap_2d(__VA_ARGS__)) return QLORA_ERR_CUDA;             \
  } while (0)

// T = X A (fp32, split partials) then T_save / bf16(scale T).
qlora_status lora_down_T(const uint16_t* X, const uint16_t* A, const LinearShape& s, float* part,
                         float* t_plain, uint16_t* t_scaled, cudaStream_t st) {
  CUtensorMap ta, tb;
  QL_MAP(&ta, kBF16, X, s.K, s.M, s.K * 2, 64, 128, kSW128);   // X K-major
  QL_MAP(&tb, kBF16, A, s.r, s.K, s.r * 2, 64, 64, kSW128);    // A as MN-major (j inner)
  int splits = 0;
  QL_TRY((run_lora_gemm<false, true, 64>(ta, tb, s.M, s.K, part, st, &splits)));
  const int64_t rows_pad = plan_split(s.M, s.K).rows_pad;
  QL_TRY(launch_pdl(k_finalize_rank, dim3(blocks_for(s.M * 64, 256)), dim3(256), 0, st, part,
                    splits, rows_pad, s.M, s.r, s.scale, t_plain, t_scaled, nullptr, nullptr,
                    nullptr));
  return QLORA_OK;
}

// A non-blocking side stream and two events per host thread and device, for the part of
// the backward that runs beside the fused dX kernel (fork and join by events, which a
// CUDA graph capture of the caller's stream follows).
struct SideStream {
  cudaStream_t st = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
// Null (and success) when `st` is being captured and the side stream does not exist yet:
// streams and events cannot be created during a capture, and the caller then runs
// everything in order on `st`.
cudaError_t side_stream(cudaStream_t st, SideStream** out) {
  thread_local SideStream side[16];
  *out = nullptr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 16) return cudaSuccess;
  SideStream& s = side[dev];
  if (!s.st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(st, &cs);
    if (e != cudaSuccess) return e;
    if (cs != cudaStreamCaptureStatusNone) return cudaSuccess;
    e = cudaStreamCreateWithFlags(&s.st, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.join, cudaEventDisableTiming);
    if (e != cudaSuccess) return e;
  }
  *out = &s;
  return cudaSuccess;
}

}  // namespace

size_t gemm_fwd_workspace(const LinearShape& s) {
  float* p;
  uint16_t* t;
  return fwd_layout(s, nullptr, &p, &t);
}

size_t gemm_bwd_workspace(const LinearShape& s) {
  float *p, *t;
  uint16_t *g, *gh, *th;
  return bwd_layout(s, nullptr, &p, &g, &gh, &th, &t);
}

qlora_status gemm_forward(const uint16_t* X, const qlora_nf4_weight& w, const uint16_t* A,
                          const uint16_t* B, const LinearShape& s, uint16_t* Y, float* T_save,
                          void* ws, cudaStream_t st) {
  float* part;
  uint16_t* ts;
  fwd_layout(s, ws, &part, &ts);
  qlora_status q = lora_down_T(X, A, s, part, T_save, ts, st);
  if (q != QLORA_OK) return q;

  CUtensorMap ta, tw, tx;
  QL_MAP(&ta, kBF16, X, s.K, s.M, s.K * 2, 64, 256, kSW128);
  QL_MAP(&tw, kBF16, B, s.N, s.r, s.N * 2, 64, 64, kSW128);   // B [r, N], MN-major chunks
  QL_MAP(&tx, kBF16, ts, 128, s.M, 256, 64, 256, kSW128);     // scale T, bf16 hi | lo
  FusedArgs a;
  a.codebook = w.codebook;
  a.codes = w.codes;
  a.c2 = w.c2;
  a.c1 = w.c1;
  a.mean = w.mean;
  a.N = s.N;
  a.K = s.K;
  a.M = s.M;
  a.ext_mmas = (s.r + 15) / 16;
  a.out = Y;
  a.out_f32 = false;
  a.out_ld = s.N;
  a.out_rows = s.N;
  a.err = device_error_word();
  // Y [M, N] for the tile stores: 32 x 32 boxes, 64-byte swizzle (N % 8 == 0, Y aligned)
  CUtensorMap to;
  QL_MAP(&to, kBF16, Y, s.N, s.M, s.N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
  QL_TRY(run_fused<Mode::kForward>(ta, tw, tx, to, a, st));
  return QLORA_OK;
}

qlora_status gemm_backward(const uint16_t* dY, const uint16_t* X, const float* T_saved,
                           const qlora_nf4_weight& w, const uint16_t* A, const uint16_t* B,
                           const LinearShape& s, uint16_t* dX, float* dA, float* dB, void* ws,
                           cudaStream_t st) {
  float *part, *tbuf;
  uint16_t *gs, *ghl, *thl;
  bwd_layout(s, ws, &part, &gs, &ghl, &thl, &tbuf);
  int splits = 0;

  // T (saved, or recomputed first: the partial buffer is then free again)
  const float* t = T_saved;
  if (!t) {
    qlora_status q = lora_down_T(X, A, s, part, tbuf, nullptr, st);
    if (q != QLORA_OK) return q;
    t = tbuf;
  }
  // G = dY B^T -> bf16(scale G) for the dX extension, bf16 hi/lo of G for dA; the same
  // launch turns T into its bf16 hi/lo pair for dB.
  {
    CUtensorMap ta, tb;
    QL_MAP(&ta, kBF16, dY, s.N, s.M, s.N * 2, 64, 128, kSW128);  // dY K-major (over n)
    QL_MAP(&tb, kBF16, B, s.N, s.r, s.N * 2, 64, 64, kSW128);    // B [r, N] K-major
    QL_TRY((run_lora_gemm<false, false, 64>(ta, tb, s.M, s.N, part, st, &splits)));
    QL_TRY(launch_pdl(k_finalize_rank, dim3(blocks_for(s.M * 64, 256)), dim3(256), 0, st, part,
                      splits, plan_split(s.M, s.N).rows_pad, s.M, s.r, s.scale, nullptr, gs, ghl,
                      t, thl));
  }

  // dX = dY W_hat + scale G A^T, and the grouped dA = scale X^T G (rows k) with
  // dB = scale T^T dY (rows n, stored [r, N]). dA and dB need G and T, not dX: with dX
  // requested they run on a side stream beside the fused dX kernel, whose persistent CTAs
  // are enqueued first and hold the SMs; the side stream's CTAs take SMs as fused CTAs
  // finish (the last, partial wave of tiles).
  CUtensorMap xa, xw, xx, xo, ga, gb, ga1, gb1;
  if (dX) {
    QL_MAP(&xa, kBF16, dY, s.N, s.M, s.N * 2, 64, 256, kSW128);
    QL_MAP(&xw, kBF16, A, s.r, s.K, s.r * 2, 64, 128, kSW128);   // A [K, r] K-major
    QL_MAP(&xx, kBF16, gs, 128, s.M, 256, 64, 256, kSW128);      // scale G, bf16 hi | lo
    // dX [M, K] for the tile stores: 32 x 32 boxes, 64-byte swizzle
    QL_MAP(&xo, kBF16, dX, s.K, s.M, s.K * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
  }
  QL_MAP(&ga, kBF16, X, s.K, s.M, s.K * 2, 64, 64, kSW128);    // X as MN-major (k inner)
  QL_MAP(&gb, kBF16, ghl, 128, s.M, 256, 64, 64, kSW128);      // G hi/lo MN-major
  QL_MAP(&ga1, kBF16, dY, s.N, s.M, s.N * 2, 64, 64, kSW128);  // dY as MN-major (n inner)
  QL_MAP(&gb1, kBF16, thl, 128, s.M, 256, 64, 64, kSW128);     // T hi/lo MN-major

  SideStream* side = nullptr;
  if (dX) QL_TRY(side_stream(st, &side));
  cudaStream_t gst = st;
  if (side) {
    QL_TRY(cudaEventRecord(side->fork, st));
    QL_TRY(cudaStreamWaitEvent(side->st, side->fork, 0));
    gst = side->st;
  }
  cudaError_t e = cudaSuccess;
  if (dX) {
    FusedArgs a;
    a.codebook = w.codebook;
    a.codes = w.codes;
    a.c2 = w.c2;
    a.c1 = w.c1;
    a.mean = w.mean;
    a.N = s.N;
    a.K = s.K;
    a.M = s.M;
    a.ext_mmas = (s.r + 15) / 16;
    a.out = dX;
    a.out_f32 = false;
    a.out_ld = s.K;
    a.out_rows = s.K;
    a.err = device_error_word();
    e = run_fused<Mode::kDgrad>(xa, xw, xx, xo, a, st);
  }
  if (e == cudaSuccess)
    e = run_lora_gemm<true, true, 128>(ga, gb, s.K, s.M, part, gst, &splits, &ga1, &gb1, s.N);
  if (e == cudaSuccess) {
    const int64_t stacked = stacked_rows(s.K, s.N);
    e = launch_pdl(k_finalize_grad, dim3(blocks_for(stacked, kGradRows)), dim3(256), 0, gst,
                   part, splits, plan_split(stacked, s.M).rows_pad,
                   static_cast<int64_t>(align_up(s.K, 128)), s.K, dA, s.N, dB, s.r, s.scale);
  }
  if (side) {  // the caller's stream continues once both branches are done (on every path)
    cudaError_t ej = cudaEventRecord(side->join, side->st);
    if (ej == cudaSuccess) ej = cudaStreamWaitEvent(st, side->join, 0);
    if (e == cudaSuccess) e = ej;
  }
  QL_TRY(e);
  return QLORA_OK;
}

// ---- column (N) sharding of W: the backward of one shard
size_t gemm_shard_g_workspace(const LinearShape& s) {
  return align_up(partial_floats(s.M, s.N, 64) * sizeof(float), 256) + 256;
}

qlora_status gemm_shard_g(const uint16_t* dY, const uint16_t* B, const LinearShape& s,
                          float* G_part, void* ws, cudaStream_t st) {
  float* part = static_cast<float*>(ws);
  CUtensorMap ta, tb;
  QL_MAP(&ta, kBF16, dY, s.N, s.M, s.N * 2, 64, 128, kSW128);  // dY K-major (over n)
  QL_MAP(&tb, kBF16, B, s.N, s.r, s.N * 2, 64, 64, kSW128);    // B [r, N] K-major
  int splits = 0;
  QL_TRY((run_lora_gemm<false, false, 64>(ta, tb, s.M, s.N, part, st, &splits)));
  QL_TRY(launch_pdl(k_finalize_rank, dim3(blocks_for(s.M * 64, 256)), dim3(256), 0, st, part,
                    splits, plan_split(s.M, s.N).rows_pad, s.M, s.r, s.scale, G_part, nullptr,
                    nullptr, nullptr, nullptr));
  return QLORA_OK;
}

size_t gemm_shard_bwd_workspace(const LinearShape& s) {
  float *p, *t;
  uint16_t *g, *gh, *th;
  return bwd_layout(s, nullptr, &p, &g, &gh, &th, &t);
}

qlora_status gemm_shard_bwd(const uint16_t* dY, const uint16_t* X, const float* T_saved,
                            const float* G, const qlora_nf4_weight& w, const uint16_t* A,
                            const uint16_t* B, const LinearShape& s, bool lora_in_dx,
                            float* dX_part, float* dA, float* dB, void* ws, cudaStream_t st) {
  float *part, *tbuf;
  uint16_t *gs, *ghl, *thl;
  bwd_layout(s, ws, &part, &gs, &ghl, &thl, &tbuf);
  const float* t = T_saved;
  if (!t) {
    qlora_status q = lora_down_T(X, A, s, part, tbuf, nullptr, st);
    if (q != QLORA_OK) return q;
    t = tbuf;
  }
  QL_TRY(launch_pdl(k_rank_from_plain, dim3(blocks_for(s.M * 64, 256)), dim3(256), 0, st, G, t,
                    s.M, s.r, s.scale, gs, ghl, thl));
  CUtensorMap xa, xw, xx, xo, ga, gb, ga1, gb1;
  if (dX_part) {
    QL_MAP(&xa, kBF16, dY, s.N, s.M, s.N * 2, 64, 256, kSW128);
    QL_MAP(&xw, kBF16, A, s.r, s.K, s.r * 2, 64, 128, kSW128);   // A [K, r] K-major
    QL_MAP(&xx, kBF16, gs, 128, s.M, 256, 64, 256, kSW128);      // scale G, bf16 hi | lo
    // fp32 dX partial sums [M, K]: 32 x 32 boxes, no swizzle
    QL_MAP(&xo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, dX_part, s.K, s.M, s.K * 4, 32, 32,
           CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  QL_MAP(&ga, kBF16, X, s.K, s.M, s.K * 2, 64, 64, kSW128);
  QL_MAP(&gb, kBF16, ghl, 128, s.M, 256, 64, 64, kSW128);
  QL_MAP(&ga1, kBF16, dY, s.N, s.M, s.N * 2, 64, 64, kSW128);
  QL_MAP(&gb1, kBF16, thl, 128, s.M, 256, 64, 64, kSW128);
  SideStream* side = nullptr;
  if (dX_part) QL_TRY(side_stream(st, &side));
  cudaStream_t gst = st;
  if (side) {
    QL_TRY(cudaEventRecord(side->fork, st));
    QL_TRY(cudaStreamWaitEvent(side->st, side->fork, 0));
    gst = side->st;
  }
  cudaError_t e = cudaSuccess;
  if (dX_part) {
    FusedArgs a;
    a.codebook = w.codebook;
    a.codes = w.codes;
    a.c2 = w.c2;
    a.c1 = w.c1;
    a.mean = w.mean;
    a.N = s.N;
    a.K = s.K;
    a.M = s.M;
    a.ext_mmas = lora_in_dx ? (s.r + 15) / 16 : 0;
    a.out = nullptr;
    a.out_f32 = true;
    a.out_ld = s.K;
    a.out_rows = s.K;
    a.err = device_error_word();
    e = run_fused<Mode::kDgrad>(xa, xw, xx, xo, a, st);
  }
  int splits = 0;
  if (e == cudaSuccess)
    e = run_lora_gemm<true, true, 128>(ga, gb, s.K, s.M, part, gst, &splits, &ga1, &gb1, s.N);
  if (e == cudaSuccess) {
    const int64_t stacked = stacked_rows(s.K, s.N);
    e = launch_pdl(k_finalize_grad, dim3(blocks_for(stacked, kGradRows)), dim3(256), 0, gst,
                   part, splits, plan_split(stacked, s.M).rows_pad,
                   static_cast<int64_t>(align_up(s.K, 128)), s.K, dA, s.N, dB, s.r, s.scale);
  }
  if (side) {
    cudaError_t ej = cudaEventRecord(side->join, side->st);
    if (ej == cudaSuccess) ej = cudaStreamWaitEvent(st, side->join, 0);
    if (e == cudaSuccess) e = ej;
  }
  QL_TRY(e);
  return QLORA_OK;
}

cudaError_t launch_to_bf16(const float* src, uint16_t* dst, int64_t n, cudaStream_t st) {
  const int64_t n4 = n / 4;
  const int64_t blocks = std::min<int64_t>((n4 + 255) / 256, static_cast<int64_t>(num_sms()) * 8);
  return launch_pdl(k_to_bf16, dim3(static_cast<unsigned>(std::max<int64_t>(blocks, 1))), dim3(256),
                    0, st, reinterpret_cast<const float4*>(src), reinterpret_cast<uint2*>(dst), n4);
}

}  // namespace qlora
