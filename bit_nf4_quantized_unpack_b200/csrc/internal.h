// internal.h -- declarations shared by the library's translation units (not installed).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/qlora.h"

namespace qlora {

// ---- code tables (tables.cpp) ---------------------------------------------------
// NF4 levels as fp32 bit patterns, ascending; index 7 is the exact zero.
extern const uint32_t kNf4Bits[16];
constexpr int kT8Size = 253;  // distinct finite E4M3 values
struct Nf4Thresholds { float t[15]; };
// NF4 codes by table: bucket b = round-half-even(16 x + 16) of x in [-1, 1] (33
// buckets of width 1/16, narrower than the smallest gap between two thresholds of either
// codebook, 0.080); within bucket b the code is code[b] + (x >= thr[b]) (thr = +inf when
// no threshold falls inside the bucket; no bucket holds two).
constexpr int kBucketScale = 16;
constexpr int kCodeBuckets = 2 * kBucketScale + 1;
struct Nf4BucketTable {
  float thr[kCodeBuckets];
  uint8_t code[kCodeBuckets + 3];
};
constexpr int kCodebooks = 2;  // qlora_codebook: 0 NF4, 1 uniform 4-bit
const Nf4BucketTable& code_buckets(int codebook);
const float* codebook_levels(int codebook);
struct T8Thresholds { float t[kT8Size - 1]; };
const Nf4Thresholds& nf4_thresholds();
const T8Thresholds& t8_thresholds();
const float* t8_values();        // [253] ascending
const uint8_t* t8_codes();       // [253] E4M3 bit pattern of each entry

// ---- host helpers (api.cu) -------------------------------------------------------
void set_last_error(const char* msg);
qlora_status cuda_status(cudaError_t e);          // records the message, maps the code
int num_sms();                                     // of the current device
bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                  uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_inner,
                  uint32_t box_outer, CUtensorMapSwizzle swizzle);
int* device_error_word();                          // per-device error flag of the kernels
bool is_aligned16(const void* p);
// QLORA_ERR_DEVICE unless the current device is sm_100 class (QLORA_ERR_CUDA if it cannot
// be queried)
qlora_status check_device();
// The argument checks shared by the linear entry points (weight, M, N % 8, r, scale).
qlora_status check_linear(int64_t M, const qlora_nf4_weight& w, int r, float scale);
// CUDA events (or NULL) this thread asked to have recorded around each launch of the
// fused NF4 GEMM kernel (qlora_profile_events).
void profile_events(cudaEvent_t* before, cudaEvent_t* after);
void note_launches(int n);                         // count kernels enqueued (qlora_launch_count)

// ---- launchers (codec.cu) -------------------------------------------------------
size_t quantize_workspace_bytes(int64_t n, int64_t k);
cudaError_t launch_quantize(const void* W, bool w_bf16, int64_t n, int64_t k, int codebook,
                            uint8_t* codes, uint8_t* c2, float* c1, float* mean, void* ws,
                            cudaStream_t st);
cudaError_t launch_dequant(const qlora_nf4_weight& w, uint16_t* out, cudaStream_t st);

// ---- launchers (gemm.cu) --------------------------------------------------------
struct LinearShape { int64_t M, N, K; int r; float scale; };
cudaError_t launch_merge_lora(const qlora_nf4_weight& w, const uint16_t* A, const uint16_t* B,
                              int r, float scale, uint16_t* out, cudaStream_t st);
size_t gemm_fwd_workspace(const LinearShape& s);
size_t gemm_bwd_workspace(const LinearShape& s);
qlora_status gemm_forward(const uint16_t* X, const qlora_nf4_weight& w, const uint16_t* A,
                          const uint16_t* B, const LinearShape& s, uint16_t* Y, float* T_save,
                          void* ws, cudaStream_t st);
qlora_status gemm_backward(const uint16_t* dY, const uint16_t* X, const float* T_saved,
                           const qlora_nf4_weight& w, const uint16_t* A, const uint16_t* B,
                           const LinearShape& s, uint16_t* dX, float* dA, float* dB, void* ws,
                           cudaStream_t st);

// Column (N) sharding of W (gemm.cu): the backward of one shard, whose weight is rows
// [row0, row0 + N) of W. gemm_shard_g: G_part = dY B^T (fp32, unscaled); once G is summed
// over the shards, gemm_shard_bwd: dX_part = dY W_hat (+ scale G A^T when lora_in_dx) in
// fp32, dA = scale X^T G, dB = scale T^T dY. launch_to_bf16 rounds a summed dX.
size_t gemm_shard_g_workspace(const LinearShape& s);
qlora_status gemm_shard_g(const uint16_t* dY, const uint16_t* B, const LinearShape& s,
                          float* G_part, void* ws, cudaStream_t st);
size_t gemm_shard_bwd_workspace(const LinearShape& s);
qlora_status gemm_shard_bwd(const uint16_t* dY, const uint16_t* X, const float* T_saved,
                            const float* G, const qlora_nf4_weight& w, const uint16_t* A,
                            const uint16_t* B, const LinearShape& s, bool lora_in_dx,
                            float* dX_part, float* dA, float* dB, void* ws, cudaStream_t st);
cudaError_t launch_to_bf16(const float* src, uint16_t* dst, int64_t n, cudaStream_t st);

// ---- launchers (decode.cu) ------------------------------------------------------
constexpr int64_t kDecodeMaxM = 16;
// Workspace of the decode kernels, or 0 when they cannot run the shape (the fused GEMM
// then serves it).
size_t decode_workspace(const LinearShape& s);
qlora_status decode_forward(const uint16_t* X, const qlora_nf4_weight& w, const uint16_t* A,
                            const uint16_t* B, const LinearShape& s, uint16_t* Y,
                            float* T_save, void* ws, cudaStream_t st);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---- launchers (selftest.cu) ----------------------------------------------------
cudaError_t launch_wait_selftest(cudaStream_t st);

// ---- launchers (optim.cu) -------------------------------------------------------
// Byte offsets inside the optimizer-state buffer of n parameters (qlora_adamw_state_bytes):
// 8-bit: m codes at 0, v codes at off_vc, m absmax at off_ma, v absmax at off_va;
// 32-bit: m at 0, v at off_vc.
struct AdamwStateLayout { size_t off_vc, off_ma, off_va, total; };
AdamwStateLayout adamw_state_layout(int64_t n, int state_bits);
cudaError_t launch_adamw(float* p, uint16_t* p_bf16, const float* g, int64_t n, int state_bits,
                         void* state, const qlora_adamw_hparams& hp, cudaStream_t st);

}  // namespace qlora
