// api.cu -- the extern "C" entry points: host-side validation (nothing is launched
// when an argument is rejected), dispatch to the kernels, and host utilities.
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include "internal.h"

namespace qlora {

namespace {
thread_local char g_last_error[256] = "";
thread_local cudaEvent_t g_prof_before = nullptr;
thread_local cudaEvent_t g_prof_after = nullptr;
std::atomic<unsigned long long> g_launches{0};

// Per-device error word written by kernels whose bounded waits ran out.
__device__ int g_device_error;

constexpr int kMaxDevices = 64;
int* g_err_ptr[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};
int g_cc_major[kMaxDevices] = {};
std::mutex g_dev_mu;

bool device_info(int* dev_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    set_last_error(e != cudaSuccess ? cudaGetErrorString(e) : "device index out of range");
    return false;
  }
  std::lock_guard<std::mutex> lock(g_dev_mu);
  if (!g_err_ptr[dev]) {
    int sms = 0, major = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
      set_last_error("cudaDeviceGetAttribute failed");
      return false;
    }
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_device_error);
    if (e != cudaSuccess) {
      set_last_error(cudaGetErrorString(e));
      return false;
    }
    g_sms[dev] = sms;
    g_cc_major[dev] = major;
    g_err_ptr[dev] = static_cast<int*>(p);
  }
  *dev_out = dev;
  return true;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}


}  // namespace

bool is_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

namespace {
bool aligned16(const void* p) { return is_aligned16(p); }

// Common checks of a quantized weight.
qlora_status check_weight(const qlora_nf4_weight& w) {
  if (!w.codes || !w.c2 || !w.c1 || !w.mean) return QLORA_ERR_INVALID_ARG;
  if (w.codebook < 0 || w.codebook >= kCodebooks) return QLORA_ERR_INVALID_ARG;
  if (w.n_out < 1 || w.k_in < 64 || w.k_in % 64 != 0) return QLORA_ERR_SHAPE;
  if (w.n_out > (int64_t{1} << 31) || w.k_in > (int64_t{1} << 31)) return QLORA_ERR_SHAPE;
  if (!aligned16(w.codes) || !aligned16(w.c2) || !aligned16(w.c1) || !aligned16(w.mean))
    return QLORA_ERR_ALIGN;
  return QLORA_OK;
}

}  // namespace

qlora_status check_device() {
  int dev = 0;
  if (!device_info(&dev)) return QLORA_ERR_CUDA;
  if (g_cc_major[dev] != 10) {
    set_last_error("the kernels are built for sm_100a (B200 class)");
    return QLORA_ERR_DEVICE;
  }
  return QLORA_OK;
}

// Shape checks of the linear layer (forward and backward share them).
qlora_status check_linear(int64_t M, const qlora_nf4_weight& w, int r, float scale) {
  qlora_status q = check_weight(w);
  if (q != QLORA_OK) return q;
  if (M < 0 || M > (int64_t{1} << 31)) return QLORA_ERR_SHAPE;
  if (w.n_out % 8 != 0) return QLORA_ERR_SHAPE;  // 16-byte rows for the bf16 operands
  if (r < 8 || r > 64 || r % 8 != 0) return QLORA_ERR_INVALID_ARG;
  if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f) return QLORA_ERR_INVALID_ARG;
  return QLORA_OK;
}

void set_last_error(const char* msg) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s", msg ? msg : "");
}

qlora_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return QLORA_OK;
  set_last_error(cudaGetErrorString(e));
  return QLORA_ERR_CUDA;
}

int num_sms() {
  int dev = 0;
  if (!device_info(&dev)) return 148;
  return g_sms[dev] > 0 ? g_sms[dev] : 148;
}

void note_launches(int n) { g_launches.fetch_add(static_cast<unsigned long long>(n), std::memory_order_relaxed); }

void profile_events(cudaEvent_t* before, cudaEvent_t* after) {
  *before = g_prof_before;
  *after = g_prof_after;
}

int* device_error_word() {
  int dev = 0;
  if (!device_info(&dev)) return nullptr;
  return g_err_ptr[dev];
}

bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                  uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                  CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (!fn) {
    set_last_error("cuTensorMapEncodeTiled is not available from the driver");
    return false;
  }
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char msg[160];
    std::snprintf(msg, sizeof(msg), "cuTensorMapEncodeTiled failed (%d) dims %llu x %llu", int(r),
                  static_cast<unsigned long long>(inner), static_cast<unsigned long long>(outer));
    set_last_error(msg);
    return false;
  }
  return true;
}

}  // namespace qlora

using namespace qlora;

extern "C" {

const char* qlora_status_str(qlora_status s) {
  switch (s) {
    case QLORA_OK: return "QLORA_OK";
    case QLORA_ERR_INVALID_ARG: return "QLORA_ERR_INVALID_ARG";
    case QLORA_ERR_SHAPE: return "QLORA_ERR_SHAPE";
    case QLORA_ERR_ALIGN: return "QLORA_ERR_ALIGN";
    case QLORA_ERR_WORKSPACE: return "QLORA_ERR_WORKSPACE";
    case QLORA_ERR_CUDA: return "QLORA_ERR_CUDA";
    case QLORA_ERR_DEVICE: return "QLORA_ERR_DEVICE";
    case QLORA_ERR_TIMEOUT: return "QLORA_ERR_TIMEOUT";
  }
  return "QLORA_ERR_UNKNOWN";
}

const char* qlora_last_error(void) { return g_last_error; }

int qlora_version(void) { return 100; }

unsigned long long qlora_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

void qlora_profile_events(void* before, void* after) {
  g_prof_before = static_cast<cudaEvent_t>(before);
  g_prof_after = static_cast<cudaEvent_t>(after);
}

qlora_status qlora_device_error(int clear) {
  int dev = 0;
  if (!device_info(&dev)) return QLORA_ERR_CUDA;
  int v = 0;
  cudaError_t e = cudaMemcpy(&v, g_err_ptr[dev], sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_status(e);
  if (clear && v != 0) {
    const int zero = 0;
    e = cudaMemcpy(g_err_ptr[dev], &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_status(e);
  }
  if (v != 0) {
    char msg[96];
    std::snprintf(msg, sizeof(msg), "a kernel wait timed out (device code %d)", v);
    set_last_error(msg);
    return QLORA_ERR_TIMEOUT;
  }
  return QLORA_OK;
}

size_t qlora_quantize_workspace_size(int64_t n_out, int64_t k_in) {
  if (n_out < 1 || k_in < 64 || k_in % 64 != 0) return 0;
  return quantize_workspace_bytes(n_out, k_in);
}

qlora_status qlora_quantize_dq(const void* W, qlora_dtype w_dtype, int64_t n_out, int64_t k_in,
                               int32_t codebook, uint8_t* codes, uint8_t* c2, float* c1,
                               float* mean, void* workspace, size_t workspace_bytes, void* stream) {
  if (codebook < 0 || codebook >= kCodebooks) return QLORA_ERR_INVALID_ARG;
  if (!W || !codes || !c2 || !c1 || !mean) return QLORA_ERR_INVALID_ARG;
  if (w_dtype != QLORA_F32 && w_dtype != QLORA_BF16) return QLORA_ERR_INVALID_ARG;
  if (n_out < 1 || k_in < 64 || k_in % 64 != 0) return QLORA_ERR_SHAPE;
  if (n_out > (int64_t{1} << 31) || k_in > (int64_t{1} << 31)) return QLORA_ERR_SHAPE;
  if (n_out * k_in / 64 > (int64_t{1} << 31)) return QLORA_ERR_SHAPE;  // the mean's exact sums
  if (!aligned16(W) || !aligned16(codes) || !aligned16(c2) || !aligned16(c1) || !aligned16(mean))
    return QLORA_ERR_ALIGN;
  if (!workspace || workspace_bytes < quantize_workspace_bytes(n_out, k_in))
    return QLORA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QLORA_ERR_ALIGN;
  qlora_status q = check_device();
  if (q != QLORA_OK) return q;
  return cuda_status(launch_quantize(W, w_dtype == QLORA_BF16, n_out, k_in, codebook, codes, c2,
                                     c1, mean, workspace, static_cast<cudaStream_t>(stream)));
}

qlora_status qlora_quantize_nf4_dq(const void* W, qlora_dtype w_dtype, int64_t n_out, int64_t k_in,
                                   uint8_t* codes, uint8_t* c2, float* c1, float* mean,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  return qlora_quantize_dq(W, w_dtype, n_out, k_in, QLORA_CODEBOOK_NF4, codes, c2, c1, mean,
                           workspace, workspace_bytes, stream);
}

qlora_status qlora_dequant(qlora_nf4_weight w, uint16_t* W_out, void* stream) {
  qlora_status q = check_weight(w);
  if (q != QLORA_OK) return q;
  if (!W_out) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(W_out)) return QLORA_ERR_ALIGN;
  q = check_device();
  if (q != QLORA_OK) return q;
  return cuda_status(launch_dequant(w, W_out, static_cast<cudaStream_t>(stream)));
}

qlora_status qlora_merge_lora(qlora_nf4_weight w, const uint16_t* A, const uint16_t* B, int r,
                              float scale, uint16_t* W_out, void* stream) {
  qlora_status q = check_linear(0, w, r, scale);
  if (q != QLORA_OK) return q;
  if (!A || !B || !W_out) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(B) || !aligned16(W_out)) return QLORA_ERR_ALIGN;
  q = check_device();
  if (q != QLORA_OK) return q;
  return cuda_status(launch_merge_lora(w, A, B, r, scale, W_out, static_cast<cudaStream_t>(stream)));
}

size_t qlora_linear_fwd_workspace_size(int64_t M, int64_t n_out, int64_t k_in, int r) {
  if (M < 0 || n_out < 1 || k_in < 64 || r < 8 || r > 64) return 0;
  const LinearShape s{M, n_out, k_in, r, 1.f};
  const size_t dec = M <= kDecodeMaxM ? decode_workspace(s) : 0;
  return dec ? dec : gemm_fwd_workspace(s);
}

qlora_status qlora_linear_fwd(const uint16_t* X, int64_t M, qlora_nf4_weight w, const uint16_t* A,
                              const uint16_t* B, int r, float scale, uint16_t* Y, float* T_save,
                              void* workspace, size_t workspace_bytes, void* stream) {
  qlora_status q = check_linear(M, w, r, scale);
  if (q != QLORA_OK) return q;
  if (M == 0) return QLORA_OK;  // empty batch: nothing to compute (X, Y may be NULL)
  if (!X || !A || !B || !Y) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(Y) ||
      (T_save && !aligned16(T_save)))
    return QLORA_ERR_ALIGN;
  const LinearShape s{M, w.n_out, w.k_in, r, scale};
  // M <= 16 takes the decode kernels, unless they cannot run the shape
  const size_t dec = M <= kDecodeMaxM ? decode_workspace(s) : 0;
  const size_t need = dec ? dec : gemm_fwd_workspace(s);
  if (!workspace || workspace_bytes < need) return QLORA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QLORA_ERR_ALIGN;
  q = check_device();
  if (q != QLORA_OK) return q;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dec ? decode_forward(X, w, A, B, s, Y, T_save, workspace, st)
             : gemm_forward(X, w, A, B, s, Y, T_save, workspace, st);
}

size_t qlora_linear_bwd_workspace_size(int64_t M, int64_t n_out, int64_t k_in, int r) {
  if (M < 0 || n_out < 1 || k_in < 64 || r < 8 || r > 64) return 0;
  return gemm_bwd_workspace(LinearShape{M, n_out, k_in, r, 1.f});
}

qlora_status qlora_linear_bwd(const uint16_t* dY, const uint16_t* X, const float* T_saved,
                              int64_t M, qlora_nf4_weight w, const uint16_t* A, const uint16_t* B,
                              int r, float scale, uint16_t* dX, float* dA, float* dB,
                              void* workspace, size_t workspace_bytes, void* stream) {
  qlora_status q = check_linear(M, w, r, scale);
  if (q != QLORA_OK) return q;
  if (!dA || !dB) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(dA) || !aligned16(dB)) return QLORA_ERR_ALIGN;
  const LinearShape s{M, w.n_out, w.k_in, r, scale};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (M > 0) {
    if (!dY || !X || !A || !B) return QLORA_ERR_INVALID_ARG;
    if (!aligned16(dY) || !aligned16(X) || !aligned16(A) || !aligned16(B) ||
        (dX && !aligned16(dX)) || (T_saved && !aligned16(T_saved)))
      return QLORA_ERR_ALIGN;
  }
  if (M == 0) {  // empty batch: the gradients of A and B are zero
    q = check_device();
    if (q != QLORA_OK) return q;
    cudaError_t e = cudaMemsetAsync(dA, 0, static_cast<size_t>(w.k_in) * r * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dB, 0, static_cast<size_t>(w.n_out) * r * 4, st);
    return cuda_status(e);
  }
  if (!workspace || workspace_bytes < gemm_bwd_workspace(s)) return QLORA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QLORA_ERR_ALIGN;
  q = check_device();
  if (q != QLORA_OK) return q;
  return gemm_backward(dY, X, T_saved, w, A, B, s, dX, dA, dB, workspace, st);
}

// ---- column (N) sharding of W

qlora_status qlora_shard_rows(int64_t n_out, int64_t k_in, int32_t world, int32_t rank,
                              int64_t* row0, int64_t* rows) {
  if (!row0 || !rows || world < 1 || rank < 0 || rank >= world) return QLORA_ERR_INVALID_ARG;
  if (n_out < 1 || k_in < 64 || k_in % 64 != 0 || n_out % 8 != 0) return QLORA_ERR_SHAPE;
  // a cut at row n keeps the shard's 256-constant blocks of c1 whole and its c1 16-byte
  // aligned when n * k_in is a multiple of 4 * 256 * 64 = 65536; rows come in multiples of 8
  int64_t g = k_in, h = 65536;
  while (h) {
    const int64_t t = g % h;
    g = h;
    h = t;
  }
  // g divides 65536, so the rows per cut are a power of two; at least 8
  const int64_t unit = std::max<int64_t>(65536 / g, 8);
  const int64_t units = n_out / unit;
  if (units < world) {
    set_last_error("qlora_shard_rows: fewer whole cut units than shards");
    return QLORA_ERR_SHAPE;
  }
  const int64_t u0 = units * rank / world, u1 = units * (rank + 1) / world;
  *row0 = u0 * unit;
  *rows = (rank == world - 1) ? n_out - *row0 : (u1 - u0) * unit;
  return QLORA_OK;
}

qlora_status qlora_shard_weight(qlora_nf4_weight w, int64_t row0, int64_t rows,
                                qlora_nf4_weight* out) {
  if (!out) return QLORA_ERR_INVALID_ARG;
  qlora_status q = check_weight(w);
  if (q != QLORA_OK) return q;
  if (row0 < 0 || rows < 8 || rows % 8 != 0 || row0 + rows > w.n_out) return QLORA_ERR_SHAPE;
  if ((row0 * w.k_in) % 65536 != 0) {
    set_last_error("qlora_shard_weight: row0 * k_in must be a multiple of 65536");
    return QLORA_ERR_SHAPE;
  }
  *out = w;
  out->codes = w.codes + row0 * (w.k_in / 2);
  out->c2 = w.c2 + row0 * (w.k_in / 64);
  out->c1 = w.c1 + row0 * w.k_in / 16384;
  out->n_out = rows;
  return QLORA_OK;
}

size_t qlora_linear_bwd_shard_g_workspace_size(int64_t M, int64_t n_shard, int r) {
  if (M < 0 || n_shard < 8 || r < 8 || r > 64) return 0;
  return gemm_shard_g_workspace(LinearShape{M, n_shard, 64, r, 1.f});
}

qlora_status qlora_linear_bwd_shard_g(const uint16_t* dY, int64_t M, int64_t n_shard,
                                      const uint16_t* B, int r, float* G_part, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  if (M < 0 || M > (int64_t{1} << 31) || n_shard < 8 || n_shard % 8 != 0) return QLORA_ERR_SHAPE;
  if (r < 8 || r > 64 || r % 8 != 0) return QLORA_ERR_INVALID_ARG;
  if (!G_part) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(G_part)) return QLORA_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (M == 0) return QLORA_OK;
  if (!dY || !B) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(dY) || !aligned16(B)) return QLORA_ERR_ALIGN;
  const LinearShape s{M, n_shard, 64, r, 1.f};
  if (!workspace || workspace_bytes < gemm_shard_g_workspace(s)) return QLORA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QLORA_ERR_ALIGN;
  qlora_status q = check_device();
  if (q != QLORA_OK) return q;
  return gemm_shard_g(dY, B, s, G_part, workspace, st);
}

size_t qlora_linear_bwd_shard_workspace_size(int64_t M, int64_t n_shard, int64_t k_in, int r) {
  if (M < 0 || n_shard < 1 || k_in < 64 || r < 8 || r > 64) return 0;
  return gemm_shard_bwd_workspace(LinearShape{M, n_shard, k_in, r, 1.f});
}

qlora_status qlora_linear_bwd_shard(const uint16_t* dY, const uint16_t* X, const float* T_saved,
                                    const float* G, int64_t M, qlora_nf4_weight w,
                                    const uint16_t* A, const uint16_t* B, int r, float scale,
                                    int32_t lora_in_dx, float* dX_part, float* dA, float* dB,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  qlora_status q = check_linear(M, w, r, scale);
  if (q != QLORA_OK) return q;
  if (!dA || !dB) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(dA) || !aligned16(dB)) return QLORA_ERR_ALIGN;
  const LinearShape s{M, w.n_out, w.k_in, r, scale};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (M == 0) {  // empty batch: zero gradients, nothing to add to dX
    q = check_device();
    if (q != QLORA_OK) return q;
    cudaError_t e = cudaMemsetAsync(dA, 0, static_cast<size_t>(w.k_in) * r * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dB, 0, static_cast<size_t>(w.n_out) * r * 4, st);
    return cuda_status(e);
  }
  if (!dY || !X || !G || !A || !B) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(dY) || !aligned16(X) || !aligned16(G) || !aligned16(A) || !aligned16(B) ||
      (dX_part && !aligned16(dX_part)) || (T_saved && !aligned16(T_saved)))
    return QLORA_ERR_ALIGN;
  if (!workspace || workspace_bytes < gemm_shard_bwd_workspace(s)) return QLORA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QLORA_ERR_ALIGN;
  q = check_device();
  if (q != QLORA_OK) return q;
  return gemm_shard_bwd(dY, X, T_saved, G, w, A, B, s, lora_in_dx != 0, dX_part, dA, dB,
                        workspace, st);
}

qlora_status qlora_f32_to_bf16(const float* src, uint16_t* dst, int64_t n, void* stream) {
  if (n < 0 || n % 4 != 0) return QLORA_ERR_SHAPE;
  if (n == 0) return QLORA_OK;
  if (!src || !dst) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(src) || !aligned16(dst)) return QLORA_ERR_ALIGN;
  qlora_status q = check_device();
  if (q != QLORA_OK) return q;
  return cuda_status(launch_to_bf16(src, dst, n, static_cast<cudaStream_t>(stream)));
}

qlora_status qlora_selftest_wait_timeout(void* stream) {
  qlora_status q = check_device();
  if (q != QLORA_OK) return q;
  return cuda_status(launch_wait_selftest(static_cast<cudaStream_t>(stream)));
}

size_t qlora_adamw_state_bytes(int64_t n, int32_t state_bits) {
  if (n < 0 || (state_bits != 8 && state_bits != 32)) return 0;
  return adamw_state_layout(n, state_bits).total;
}

qlora_status qlora_adamw_step(float* p, uint16_t* p_bf16, const float* g, int64_t n,
                              int32_t state_bits, void* state, size_t state_bytes,
                              qlora_adamw_hparams hp, void* stream) {
  if (n < 0 || (state_bits != 8 && state_bits != 32) || hp.step < 1) return QLORA_ERR_INVALID_ARG;
  auto finite = [](float x) { return x == x && x < 3.5e38f && x > -3.5e38f; };
  if (!finite(hp.lr) || !finite(hp.eps) || !finite(hp.weight_decay) || !finite(hp.beta1) ||
      !finite(hp.beta2) || hp.lr < 0.f || !(hp.eps > 0.f) || hp.weight_decay < 0.f ||
      hp.beta1 < 0.f || !(hp.beta1 < 1.f) || hp.beta2 < 0.f || !(hp.beta2 < 1.f))
    return QLORA_ERR_INVALID_ARG;
  if (n == 0) return QLORA_OK;
  if (!p || !g || !state) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(p) || !aligned16(g) || !aligned16(state) || (p_bf16 && !aligned16(p_bf16)))
    return QLORA_ERR_ALIGN;
  if (state_bytes < adamw_state_layout(n, state_bits).total) return QLORA_ERR_WORKSPACE;
  qlora_status q = check_device();
  if (q != QLORA_OK) return q;
  return cuda_status(launch_adamw(p, p_bf16, g, n, state_bits, state, hp,
                                  static_cast<cudaStream_t>(stream)));
}

qlora_status qlora_paged_alloc(void** out, size_t bytes) {
  if (!out || bytes == 0) return QLORA_ERR_INVALID_ARG;
  *out = nullptr;
  void* ptr = nullptr;
  cudaError_t e = cudaMallocManaged(&ptr, bytes, cudaMemAttachGlobal);
  if (e != cudaSuccess) return cuda_status(e);
  e = cudaMemset(ptr, 0, bytes);  // a fresh optimizer state is all zeros
  if (e != cudaSuccess) {
    cudaFree(ptr);
    return cuda_status(e);
  }
  e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    cudaFree(ptr);
    return cuda_status(e);
  }
  *out = ptr;
  return QLORA_OK;
}

qlora_status qlora_paged_free(void* ptr) {
  if (!ptr) return QLORA_OK;
  return cuda_status(cudaFree(ptr));
}

qlora_status qlora_paged_prefetch(const void* ptr, size_t bytes, int32_t to_device, void* stream) {
  if (!ptr) return QLORA_ERR_INVALID_ARG;
  if (bytes == 0) return QLORA_OK;
  int dev = cudaCpuDeviceId;
  if (to_device) {
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e);
  }
  return cuda_status(cudaMemPrefetchAsync(ptr, bytes, dev, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
