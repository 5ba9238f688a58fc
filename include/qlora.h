/*
 * qlora.h -- C ABI of a B200 (sm_100a) library for the QLoRA linear layer.
 *
 * The layer (page "QLoRA", itwiki.kr, section "계산 방식" / computation, and page
 * "quantization", minnong511 blog, section "QLoRA에서 학습은 어떻게 되는 걸까?"):
 *
 *     Y = X * doubleDequant(c1, c2, W_NF4)^T + (alpha / r) * (X * A) * B
 *
 * with W stored as 4-bit NormalFloat codes in blocks of 64 weights (itwiki "QLoRA",
 * section "4비트 NormalFloat(NF4)"), the per-block absmax constants double-quantized
 * to FP8 E4M3 codes c2 in blocks of 256 after subtracting one mean per tensor, with
 * one fp32 constant c1 per 256-block (itwiki "QLoRA", section "이중 양자화").
 * The backward produces dX through the frozen quantized W and the LoRA gradients
 * dA and dB only (itwiki "QLoRA", computation section; minnong511 "quantization",
 * section on why a 4-bit base model can be trained).
 *
 * Conventions shared by every entry point:
 *  - Matrices are row-major. W is N x K (out x in) with K % 64 == 0. X is M x K,
 *    Y is M x N, A is K x r, B is r x N.
 *  - bf16 data is passed as uint16_t bit patterns.
 *  - Every pointer argument named "device" is CUDA device memory owned by the
 *    caller. The library allocates, frees and keeps no device memory, with two
 *    exceptions declared below: the fixed static scratch array of
 *    qlora_linear_fwd_decode_static, and qlora_paged_alloc, which exists to allocate
 *    unified memory for optimizer states. Other scratch space comes from the caller
 *    through (workspace, workspace_bytes); the matching *_workspace_size query says
 *    how much.
 *  - Device pointers must be 16-byte aligned (QLORA_ERR_ALIGN otherwise).
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream)
 *    and runs asynchronously. Argument errors are detected on the host before
 *    anything is launched; then nothing is enqueued and an error code is
 *    returned. QLORA_ERR_CUDA reports a failed launch; qlora_last_error() gives
 *    the CUDA message. Device-side faults surface at the caller's next
 *    synchronisation, as with any CUDA call.
 *  - All entry points are thread-safe; calls on different streams may overlap,
 *    provided their outputs and workspaces do not alias.
 *
 * Storage of a quantized weight W [N, K] (all device memory):
 *    codes : uint8 [N*K/2]   byte b = code(2b) | code(2b+1) << 4 (row-major order)
 *    c2    : uint8 [N*K/64]  E4M3 bit pattern of each block constant after
 *                            mean subtraction and 256-block scaling
 *    c1    : float [ceil(N*K/16384)] absmax of each 256-block of centred constants
 *    mean  : float [1]       mean of all N*K/64 block absmax values
 * Double dequantization of block j (flat index, 64 weights each):
 *    s_j = fl32(fl32(T8[c2_j] * c1[j/256]) + mean),  T8[e] = fl32(e4m3(e) / 448)
 *    W_hat = bf16_rn(fl32(NF4[code] * s_j))
 */
#ifndef QLORA_H
#define QLORA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = 1, /* null pointer, unknown dtype, r or scale out of range */
  QLORA_ERR_SHAPE = 2,       /* unsupported sizes (K % 64 != 0, negative sizes, ...) */
  QLORA_ERR_ALIGN = 3,       /* a device pointer is not 16-byte aligned */
  QLORA_ERR_WORKSPACE = 4,   /* workspace NULL or smaller than the size query */
  QLORA_ERR_CUDA = 5,        /* a CUDA call failed; see qlora_last_error() */
  QLORA_ERR_DEVICE = 6,      /* current device is not sm_100 (B200 class) */
  QLORA_ERR_TIMEOUT = 7      /* a kernel's bounded wait ran out (qlora_device_error) */
} qlora_status;

typedef enum { QLORA_F32 = 0, QLORA_BF16 = 1 } qlora_dtype;

/* A quantized weight as produced by qlora_quantize_nf4_dq (device pointers). */
/*
 * The 4-bit codebook L of a stored weight. NF4 is the method's own; UNIFORM4 is the
 * comparison codebook of the same itwiki section (16 evenly spaced levels on [-1, 1],
 * "uniform 4-bit, same method"), which goes through the same blocking, nearest-level
 * search, double quantization and kernels.
 */
typedef enum { QLORA_CODEBOOK_NF4 = 0, QLORA_CODEBOOK_UNIFORM4 = 1 } qlora_codebook;

typedef struct {
  const uint8_t *codes;
  const uint8_t *c2;
  const float *c1;
  const float *mean;
  int64_t n_out;    /* N: rows (output features) */
  int64_t k_in;     /* K: columns (input features), K % 64 == 0 */
  int32_t codebook; /* qlora_codebook of the codes (0 = NF4) */
} qlora_nf4_weight;

/* Human-readable name of a status code (static storage). */
const char *qlora_status_str(qlora_status status);

/* Message of the last CUDA error seen by this thread inside the library, or "". */
const char *qlora_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int qlora_version(void);

/*
 * qlora_device_error: synchronous check of the current device's error word. Every
 * wait inside the kernels is bounded (2 s); a wait that runs out records a code
 * there and the kernel drains its copies, frees its tensor memory and exits
 * without writing its outputs. Returns QLORA_ERR_TIMEOUT when a code is set (and
 * clears it when `clear` != 0), QLORA_OK otherwise. Blocks until the device copy of
 * the word is read (a synchronous cudaMemcpy on the legacy stream).
 */
qlora_status qlora_device_error(int clear);

/*
 * qlora_profile_events: measurement aid. For the calling thread, record the CUDA
 * events `before` and `after` (cudaEvent_t, or NULL to stop) on the launch stream
 * immediately before and after each launch of the fused NF4 tensor-core GEMM
 * (forward or dX), so that cudaEventElapsedTime gives that kernel's own duration.
 * The events are owned by the caller; each later launch re-records them.
 */
void qlora_profile_events(void *before, void *after);

/*
 * qlora_launch_count: number of kernel launches this library has issued in this
 * process, on all streams and devices (each launch is counted when it is enqueued).
 * The difference of two readings is the number of the library's kernels between them.
 */
unsigned long long qlora_launch_count(void);

/*
 * qlora_nf4_table: writes the 16 NF4 levels (fp32, ascending, NF4[7] == 0) that the
 * kernels use, to host memory `out16`. Host-only, needs no GPU.
 * Definition: itwiki "QLoRA", section "4비트 NormalFloat(NF4)": N(0,1) quantiles at
 * evenly spaced probabilities from 0.9677083 down to 1/2, 8 positive and 7
 * negative plus an exact zero, normalised by the largest magnitude.
 */
void qlora_nf4_table(float *out16);

/*
 * qlora_nf4_thresholds: writes the 15 decision thresholds of the NF4 code search to
 * host memory `out15`: code(x) = number of i with x >= out15[i], for every fp32 x in
 * [-1, 1]. They reproduce argmin_i fl32(|x - NF4[i]|) with ties to the lower index
 * exactly. Host-only.
 */
void qlora_nf4_thresholds(float *out15);

/*
 * qlora_nf4_code_buckets: the table form of the same code search that the
 * quantization kernel uses, to host memory. For fp32 x in [-1, 1] let
 * b = round-half-even(16 x + 16) (0 <= b <= 32: 33 buckets of width 1/16, each
 * holding at most one threshold); then
 * code(x) = code33[b] + (x >= thr33[b] ? 1 : 0), with thr33[b] = +inf when no
 * threshold lies in bucket b. Either pointer may be NULL. Host-only.
 */
void qlora_nf4_code_buckets(float *thr33, uint8_t *code33);

/*
 * The same three tables for any codebook (qlora_codebook): its 16 levels (fp32,
 * ascending), its 15 exact decision thresholds, and its 33-bucket code table. Null
 * output pointers are skipped. Returns 0, or -1 for an unknown codebook. Host-only.
 */
int qlora_codebook_tables(int32_t codebook, float *levels16, float *thr15, float *bucket_thr33,
                          uint8_t *bucket_code33);

/*
 * qlora_fp8_thresholds: the same for the 253-entry double-quantization table T8
 * (distinct finite E4M3 values / 448, ascending): 252 thresholds to host memory
 * `out252`; also writes T8 itself to `t8_out253` and the E4M3 bit pattern of each
 * entry to `codes_out253` when those are not NULL. Host-only.
 */
void qlora_fp8_thresholds(float *out252, float *t8_out253, uint8_t *codes_out253);

/* Device bytes of workspace qlora_quantize_nf4_dq needs for an N x K weight. */
size_t qlora_quantize_workspace_size(int64_t n_out, int64_t k_in);

/*
 * qlora_quantize_nf4_dq: quantize W [n_out, k_in] (device, fp32 or bf16 per
 * `w_dtype`) to NF4 with double-quantized constants.
 * Steps (itwiki "QLoRA", NF4 and double-quantization sections):
 *   1. per 64-block absmax a_j = max |w|; x = fl32(w / a_j) (x = 0 when a_j = 0);
 *      code = nearest NF4 level (ties to the lower index); two codes per byte.
 *   2. mean = the arithmetic mean of all a_j, formed exactly (integer sums of the
 *      significands per exponent, so it does not depend on the summation order or
 *      the range of the constants) and rounded once to fp32, to nearest, ties to even.
 *   3. per 256-block of centred constants cc_j = fl32(a_j - mean):
 *      c1 = max |cc|; y = fl32(cc_j / c1) (0 when c1 = 0); c2_j = E4M3 bit pattern
 *      of the nearest T8 entry (ties to the lower index).
 * Outputs (device): codes [N*K/2], c2 [N*K/64], c1 [ceil(N*K/16384)], mean [1].
 * Workspace: at least qlora_quantize_workspace_size(n_out, k_in) bytes (device).
 * Errors: QLORA_ERR_SHAPE unless n_out >= 1, k_in >= 64, k_in % 64 == 0 and
 *         n_out * k_in <= 2^37 (at most 2^31 blocks);
 *         QLORA_ERR_INVALID_ARG for a NULL pointer or unknown dtype.
 * The workspace also holds, after the absmax array, the accumulators of the mean (an
 * fp64 sum, the exponent range and a CTA count: four 64-bit words); the call clears
 * them with a small kernel on `stream` before the level-1 kernel adds to them.
 * Inputs must be finite.
 */
qlora_status qlora_quantize_nf4_dq(const void *W, qlora_dtype w_dtype, int64_t n_out,
                                   int64_t k_in, uint8_t *codes, uint8_t *c2, float *c1,
                                   float *mean, void *workspace, size_t workspace_bytes,
                                   void *stream);

/*
 * qlora_quantize_dq: qlora_quantize_nf4_dq with the 4-bit codebook chosen by `codebook`
 * (qlora_codebook). The nearest-level search uses that codebook's levels; everything
 * else (blocks, absmax, double quantization, storage) is the same. The weight it
 * describes must carry the same codebook in qlora_nf4_weight.codebook.
 * Errors: those of qlora_quantize_nf4_dq, and QLORA_ERR_INVALID_ARG for an unknown
 * codebook.
 */
qlora_status qlora_quantize_dq(const void *W, qlora_dtype w_dtype, int64_t n_out, int64_t k_in,
                               int32_t codebook, uint8_t *codes, uint8_t *c2, float *c1,
                               float *mean, void *workspace, size_t workspace_bytes,
                               void *stream);

/*
 * qlora_dequant: W_out [n_out, k_in] bf16 (device) = doubleDequant(c1, c2, W_NF4)
 * (itwiki "QLoRA", computation section; formula in the storage notes above), with the
 * levels of the weight's codebook.
 * Bit-exact with the definition. No workspace.
 */
qlora_status qlora_dequant(qlora_nf4_weight w, uint16_t *W_out, void *stream);

/*
 * qlora_merge_lora (merge_and_unload): W_out [n_out, k_in] bf16 (device) =
 * bf16(W_hat + scale (A B)^T), W_hat = doubleDequant(c1, c2, W_NF4). After training, the
 * base is dequantized to BF16 and the LoRA term added with its alpha/r scale (blog
 * "QLoRA", irregular6612, sections "학습 → 추론 파이프라인 (실무)" and
 * "재양자화 시 주의사항"; itwiki "QLoRA", section "한계와 주의점").
 *   A [k_in, r] bf16 device, B [r, n_out] bf16 device (the layout of qlora_linear_fwd).
 * Arithmetic: (A B)^T in fp32 on the tensor cores, then fl32(scale x it + W_hat) in one
 * fused multiply-add, rounded to bf16. It equals the exactly rounded sum except where that sum lies
 * within the fp32 error of a bf16 rounding boundary (then it may differ by one bf16 ulp).
 * Errors: as qlora_linear_fwd for the weight, r and scale (n_out % 8 == 0, r in
 * {8, 16, ..., 64}); QLORA_ERR_ALIGN unless A, B and W_out are 16-byte aligned.
 * No workspace.
 */
qlora_status qlora_merge_lora(qlora_nf4_weight w, const uint16_t *A, const uint16_t *B, int r,
                              float scale, uint16_t *W_out, void *stream);

/* Device bytes of workspace qlora_linear_fwd needs (0 < r <= 64, r % 8 == 0). */
size_t qlora_linear_fwd_workspace_size(int64_t M, int64_t n_out, int64_t k_in, int r);

/*
 * qlora_linear_fwd: Y [M, N] bf16 = bf16(X W_hat^T + scale (X A) B), fp32 accumulation.
 * (itwiki "QLoRA", computation section, with the alpha/r scale of minnong511
 * "quantization": scale = alpha / r.)
 *   X      [M, K] bf16 device        A [K, r] bf16 device     B [r, N] bf16 device
 *   Y      [M, N] bf16 device (written)
 *   T_save [M, r] fp32 device or NULL: when given, receives T = X A (unscaled) for
 *          the backward.
 * M >= 0 (M == 0 enqueues nothing and X, Y may be NULL); r in {8, 16, ..., 64}. M <= 16 runs the decode
 * (GEMV) kernels, larger M the fused tensor-core GEMM; both dequantize W in
 * registers without writing it to memory. The decode kernels add the partial products
 * of T = X A with fp32 atomics, so T (and through it Y) may differ in the last bits from
 * run to run; shapes they cannot run (a split's columns of X must fit 48 KB of shared
 * memory, at most 148 splits) go to the fused GEMM.
 */
qlora_status qlora_linear_fwd(const uint16_t *X, int64_t M, qlora_nf4_weight w,
                              const uint16_t *A, const uint16_t *B, int r, float scale,
                              uint16_t *Y, float *T_save, void *workspace,
                              size_t workspace_bytes, void *stream);

/*
 * qlora_linear_fwd_decode_static: the decode forward (0 <= M <= 16 tokens) of
 * qlora_linear_fwd, for callers that cannot allocate device memory when they run the
 * layer: a runtime that plans all device memory once at start-up and forbids later
 * allocation, or a token-by-token decode loop that must not pay the implicit device
 * synchronisation of cudaMalloc. It takes no workspace. The method's pages have no
 * counterpart of this entry point; it is a deployment convenience.
 *   Arguments, layouts and results are those of qlora_linear_fwd with M <= 16.
 *   Scratch: a fixed 4 MiB array in device memory inside this library, which every
 *   GPU that loads the library holds until the process exits. A call splits K into
 *   s ranges and needs
 *       align256(s * ceil(N / 16) * 16 * M * 4) + align256(M * r * 4)
 *       + align256(4 * ceil(N / 16) + 4)  bytes
 *   for fp32 partial sums, T and the arrival counters. It takes the number of splits
 *   its planner prefers when that fits, else the best that fits. The fewest splits it can
 *   run is ceil(ceil(K / 256) / u) with u = 142, 71, 47, 35, 28, 23, 20, 17, 15, 14, 12,
 *   11, 10, 10, 9, 8 for M = 1 .. 16 (a split's columns of X are staged in at most 80 KB
 *   of shared memory); when even that does not fit the array, the call is rejected with
 *   QLORA_ERR_WORKSPACE (qlora_last_error() gives the shape), and M > 16 with
 *   QLORA_ERR_SHAPE. Argument errors are checked as in qlora_linear_fwd and give its
 *   status codes.
 *   The first call on each device, and the first after that device's context changes
 *   (a cudaDeviceReset, for instance), looks up the array's device address with the
 *   device current and caches it; make that first call before any stream capture.
 *   Every call uses the same array: the set-up kernel of each call clears what must
 *   start at zero, and the partial sums are written before they are read. Calls whose
 *   kernels overlap on the GPU (different streams, or different host threads on one
 *   device) race on it: issue them in order on one stream.
 *   The function itself allocates nothing (no cudaMalloc, no cudaFree).
 */
qlora_status qlora_linear_fwd_decode_static(const uint16_t *X, int64_t M, qlora_nf4_weight w,
                                            const uint16_t *A, const uint16_t *B, int r,
                                            float scale, uint16_t *Y, float *T_save,
                                            void *stream);

/* Device bytes of workspace qlora_linear_bwd needs. */
size_t qlora_linear_bwd_workspace_size(int64_t M, int64_t n_out, int64_t k_in, int r);

/*
 * qlora_linear_bwd: gradients of qlora_linear_fwd for the upstream gradient dY.
 *   G  = dY B^T                         [M, r]
 *   dX = bf16(dY W_hat + scale G A^T)   [M, K] bf16 device, or NULL to skip
 *   dA = scale X^T G                    [K, r] fp32 device (overwritten)
 *   dB = scale T^T dY                   [r, N] fp32 device (overwritten)
 * T_saved [M, r] fp32 device is T = X A from the forward, or NULL to recompute it.
 * The quantized W is frozen: no gradient for it (itwiki "QLoRA", computation
 * section; minnong511 "quantization": W is not updated, A and B get gradients).
 * M == 0 writes zeros to dA and dB (dY, X, dX may be NULL).
 */
qlora_status qlora_linear_bwd(const uint16_t *dY, const uint16_t *X, const float *T_saved,
                              int64_t M, qlora_nf4_weight w, const uint16_t *A,
                              const uint16_t *B, int r, float scale, uint16_t *dX,
                              float *dA, float *dB, void *workspace,
                              size_t workspace_bytes, void *stream);

/*
 * Column (N) sharding of W across GPUs. The layer's backward (itwiki "QLoRA", section
 * "계산 방식": dX flows to the previous layer, gradients only for A and B) splits along
 * the output features: a shard holds rows [row0, row0 + n_shard) of the quantized W and
 * the matching columns of B, dY and Y, while X, A and T are whole on every shard. Then
 *   Y_shard = X W_hat_shard^T + scale T B_shard        (qlora_linear_fwd on the shard)
 *   G       = sum over shards of dY_shard B_shard^T     (a cross-shard sum)
 *   dX      = bf16(sum over shards of dY_shard W_hat_shard + scale G A^T)
 *   dA      = scale X^T G,   dB_shard = scale T^T dY_shard.
 * One step of a sharded backward: qlora_linear_bwd_shard_g on every shard, a sum of the
 * G_part over the shards (the caller's collective, e.g. an NCCL all-reduce), then
 * qlora_linear_bwd_shard on every shard with exactly one shard adding the LoRA term
 * (lora_in_dx = 1), a sum of the dX_part, and qlora_f32_to_bf16 of that sum.
 *
 * qlora_shard_rows: rows [*row0, *row0 + *rows) of an n_out x k_in weight for shard `rank`
 * of `world`: near-equal parts cut only where row * k_in is a multiple of 65536, so that
 * each shard's 256-constant blocks of c1 are whole (the one mean stays the tensor's) and
 * its c1 stays 16-byte aligned; the last shard takes the remainder. Host only.
 * Errors: QLORA_ERR_INVALID_ARG for NULL outputs or rank outside [0, world);
 * QLORA_ERR_SHAPE when there are fewer whole cuts than shards (or n_out % 8 != 0).
 */
qlora_status qlora_shard_rows(int64_t n_out, int64_t k_in, int32_t world, int32_t rank,
                              int64_t *row0, int64_t *rows);

/*
 * qlora_shard_weight: *out = the view of rows [row0, row0 + rows) of w as a weight of its
 * own (pointers into w's buffers; nothing is copied or allocated; w keeps ownership).
 * Errors: those of the weight checks; QLORA_ERR_SHAPE unless row0 * k_in % 65536 == 0,
 * rows % 8 == 0 and the rows lie inside w. Host only.
 */
qlora_status qlora_shard_weight(qlora_nf4_weight w, int64_t row0, int64_t rows,
                                qlora_nf4_weight *out);

/* Device bytes of workspace qlora_linear_bwd_shard_g needs. */
size_t qlora_linear_bwd_shard_g_workspace_size(int64_t M, int64_t n_shard, int r);

/*
 * qlora_linear_bwd_shard_g: G_part [M, r] fp32 (device, overwritten) = dY B^T for one
 * shard's dY [M, n_shard] and B [r, n_shard] (bf16 device), unscaled.
 * Errors: QLORA_ERR_SHAPE unless n_shard >= 8, n_shard % 8 == 0, 0 <= M <= 2^31;
 * QLORA_ERR_INVALID_ARG for r outside {8, ..., 64} or NULL pointers; QLORA_ERR_ALIGN,
 * QLORA_ERR_WORKSPACE as elsewhere. M == 0 enqueues nothing.
 */
qlora_status qlora_linear_bwd_shard_g(const uint16_t *dY, int64_t M, int64_t n_shard,
                                      const uint16_t *B, int r, float *G_part, void *workspace,
                                      size_t workspace_bytes, void *stream);

/* Device bytes of workspace qlora_linear_bwd_shard needs. */
size_t qlora_linear_bwd_shard_workspace_size(int64_t M, int64_t n_shard, int64_t k_in, int r);

/*
 * qlora_linear_bwd_shard: the rest of one shard's backward, given G [M, r] fp32 (device)
 * summed over all shards.
 *   dX_part [M, K] fp32 device (overwritten), or NULL to skip:
 *           dY W_hat_shard, plus scale G A^T when lora_in_dx != 0 (set it on one shard);
 *           computed on the tensor cores like qlora_linear_bwd's dX, but left in fp32
 *           for the cross-shard sum
 *   dA [K, r] fp32 (overwritten) = scale X^T G (the same on every shard)
 *   dB [r, n_shard] fp32 (overwritten) = scale T^T dY_shard
 * w is the shard's weight (qlora_shard_weight); dY [M, n_shard], X [M, K], A [K, r],
 * B [r, n_shard] bf16; T_saved [M, r] fp32 or NULL (recomputed from X and A).
 * Errors: as qlora_linear_bwd. M == 0 writes zeros to dA and dB.
 */
qlora_status qlora_linear_bwd_shard(const uint16_t *dY, const uint16_t *X, const float *T_saved,
                                    const float *G, int64_t M, qlora_nf4_weight w,
                                    const uint16_t *A, const uint16_t *B, int r, float scale,
                                    int32_t lora_in_dx, float *dX_part, float *dA, float *dB,
                                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * qlora_f32_to_bf16: dst[i] = bf16_rn(src[i]) for i < n (device, n % 4 == 0, 16-byte
 * aligned), e.g. dX from the sum of the shards' dX_part.
 */
qlora_status qlora_f32_to_bf16(const float *src, uint16_t *dst, int64_t n, void *stream);

/*
 * qlora_selftest_wait_timeout: a test hook for the failure path that every kernel's
 * bounded waits share (not part of the method). Enqueues on `stream` one small kernel
 * whose only wait, on an mbarrier that nothing arrives at, runs out after the library's
 * wait limit (2 s). The kernel records the timeout in the device error word and exits;
 * after the stream completes, qlora_device_error returns QLORA_ERR_TIMEOUT, and the
 * context stays usable. Errors: QLORA_ERR_DEVICE / QLORA_ERR_CUDA as the other calls.
 */
qlora_status qlora_selftest_wait_timeout(void *stream);

/*
 * ---- The optimizer step after the LoRA gradients (paged AdamW) ----
 * itwiki "QLoRA", section on paged optimizers: the optimizer states live in unified
 * memory, move to host memory when the GPU runs short and come back for the update;
 * the training example of the computation section uses optim="paged_adamw_8bit" at
 * learning rate 2e-4 and names paged_adamw_32bit beside it.
 *
 * Update of each parameter p with gradient g at step t >= 1 (AdamW: Adam with
 * decoupled weight decay), every operation one IEEE fp32 rounding, in this order:
 *   m = b1 m' + (1-b1) g          v = b2 v' + ((1-b2) g) g
 *   mh = m / bc1                  vh = v / bc2          bc_i = fl32(1 - b_i^t) (fp64 pow)
 *   p = p (1 - lr wd) - lr (mh / (sqrt(vh) + eps))
 * with (1 - b1), (1 - b2) and (1 - lr wd) formed in fp32 on the host.
 *
 * State forms (state_bits):
 *   32: m and v as fp32 arrays.
 *   8:  per block of 256 consecutive parameters one fp32 absmax per state, and per
 *       parameter one E4M3 code of the nearest entry of T8 (qlora_fp8_thresholds; ties
 *       to the lower index) to fl32(x / absmax) (0 when absmax = 0); a stored value
 *       reads back as fl32(T8[code] x absmax). The update itself uses the fp32 m and v.
 *       (The pages attribute the 8-bit states to the authors' block-wise quantization
 *       work without giving its format; this is the pages' own block-wise 8-bit float.)
 * A zero-filled state buffer is the state before the first step.
 */
typedef struct {
  float lr, beta1, beta2, eps, weight_decay;
  int64_t step; /* t of this update, 1 for the first */
} qlora_adamw_hparams;

/* Bytes of the state buffer for n parameters (state_bits 8 or 32; 0 for other values or
 * n < 0). Layout, each section starting on a 256-byte boundary: 8-bit: m codes [n],
 * v codes [n], m absmax fp32 [ceil(n/256)], v absmax fp32 [ceil(n/256)]; 32-bit: m fp32
 * [n], v fp32 [n]. */
size_t qlora_adamw_state_bytes(int64_t n, int32_t state_bits);

/*
 * qlora_adamw_step: one AdamW update of n parameters, in place.
 *   p      [n] fp32 device (or managed), the parameters (updated)
 *   p_bf16 [n] bf16 device or NULL: receives bf16_rn(p) after the update (the LoRA operand
 *          of the next forward)
 *   g      [n] fp32 device, the gradient (for the LoRA parameters: dA and dB of
 *          qlora_linear_bwd, flattened)
 *   state  device or unified memory of at least qlora_adamw_state_bytes(n, state_bits)
 *          bytes (updated)
 * n == 0 enqueues nothing. Errors: QLORA_ERR_INVALID_ARG for a NULL pointer with n > 0,
 * state_bits other than 8 or 32, step < 1, or lr, eps, weight_decay, beta outside
 * (lr >= 0, eps > 0, weight_decay >= 0, 0 <= beta < 1, all finite);
 * QLORA_ERR_WORKSPACE when state_bytes is too small; QLORA_ERR_ALIGN unless p, p_bf16,
 * g and state are 16-byte aligned. Nothing is enqueued on an error.
 */
qlora_status qlora_adamw_step(float *p, uint16_t *p_bf16, const float *g, int64_t n,
                              int32_t state_bits, void *state, size_t state_bytes,
                              qlora_adamw_hparams hp, void *stream);

/*
 * Paged optimizer states (unified memory). qlora_paged_alloc allocates `bytes` of
 * managed memory, visible to every device and the host, zero-filled (a fresh optimizer
 * state), into *out; QLORA_ERR_CUDA if the allocation fails. qlora_paged_free releases
 * it. qlora_paged_prefetch enqueues on `stream` a migration of [ptr, ptr + bytes) to the
 * current device (to_device != 0) or to host memory (to_device == 0); without it the
 * pages move on first touch. These are the only functions of the library that allocate
 * memory; they are for optimizer states, not for the layer's hot path.
 */
qlora_status qlora_paged_alloc(void **out, size_t bytes);
qlora_status qlora_paged_free(void *ptr);
qlora_status qlora_paged_prefetch(const void *ptr, size_t bytes, int32_t to_device, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H */
