// api.cu — the C ABI: argument validation, the device check, tensor-map
// encoding, the per-device error word, and dispatch to the kernels.
//
// Every call validates everything before it enqueues anything, so an error
// never leaves a partially written output.  The device check follows the
// pages' loader rule (blog.margrop.com "技术细节 §3"; app.hamidun.com
// "Какое железо и модели поддержаны"): an unsupported GPU gets a clear error,
// never a wrong result.  These kernels are sm_100a code, so "supported"
// means compute capability 10.0 exactly.
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "internal.h"
#include "ptx.cuh"

namespace svdq {

// One error word per device (the module is loaded per context).
__device__ uint32_t g_err_word;

namespace {

thread_local char t_detail[512] = "";

// Per device.  Addresses of __device__ symbols and kernel attributes belong
// to a CUDA context: after a device reset the runtime creates a new primary
// context, so they are looked up again whenever the current context's ID
// (unique for the life of the process) differs from the one they were
// taken in.
struct DeviceInfo {
  bool init = false;
  int major = 0, minor = 0, num_sms = 0;
  unsigned long long ctx_id = 0;                  // context of err_word and attrs
  uint32_t* err_word = nullptr;
  std::vector<std::pair<const void*, int>> attrs;  // (kernel, dynamic smem bytes) opted in
  cudaError_t init_err = cudaSuccess;
};

constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;
uint64_t g_timeout_ns = 2000000000ull;
int g_fault = 0;
int g_gemm_pairs = 0;
int g_pdl = 1;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_ctx_current = nullptr;
CtxGetIdFn g_ctx_id = nullptr;

template <typename Fn>
cudaError_t driver_fn(const char* name, Fn* out) {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q{};
  cudaError_t e = cudaGetDriverEntryPoint(name, &fn, cudaEnableDefault, &q);
  if (e == cudaSuccess && q != cudaDriverEntryPointSuccess) e = cudaErrorSymbolNotFound;
  if (e == cudaSuccess) *out = reinterpret_cast<Fn>(fn);
  return e;
}

// ID of the calling thread's current context (0 if none is current).
unsigned long long current_ctx_id() {
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (g_ctx_current(&c) != CUDA_SUCCESS || !c) return 0;
  if (g_ctx_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Host-side test override of the device's compute capability ("MAJOR.MINOR"),
// so that the unsupported-device path is testable without such a device.
bool forced_cc(int* major, int* minor) {
  const char* s = std::getenv("SVDQ_TEST_FORCE_CC");
  if (!s || !*s) return false;
  int a = 0, b = 0;
  if (std::sscanf(s, "%d.%d", &a, &b) != 2) return false;
  *major = a;
  *minor = b;
  return true;
}

svdq_status device_ctx(void* stream, LaunchCtx* ctx) {
  int fmaj, fmin;
  if (forced_cc(&fmaj, &fmin) && !(fmaj == 10 && fmin == 0))
    return fail(SVDQ_ERR_UNSUPPORTED_DEVICE,
                "compute capability %d.%d (forced by SVDQ_TEST_FORCE_CC): these kernels need 10.0 "
                "(sm_100a, e.g. B200)",
                fmaj, fmin);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return fail(SVDQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(SVDQ_ERR_CUDA, "device index %d too large", dev);
  DeviceInfo& d = g_dev[dev];
  std::lock_guard<std::mutex> lk(g_mu);
  if (!d.init) {
    cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (!g_encode) d.init_err = driver_fn("cuTensorMapEncodeTiled", &g_encode);
    if (!g_ctx_current && d.init_err == cudaSuccess) d.init_err = driver_fn("cuCtxGetCurrent", &g_ctx_current);
    if (!g_ctx_id && d.init_err == cudaSuccess) d.init_err = driver_fn("cuCtxGetId", &g_ctx_id);
    d.init = true;
  }
  if (!(d.major == 10 && d.minor == 0))
    return fail(SVDQ_ERR_UNSUPPORTED_DEVICE,
                "device %d has compute capability %d.%d: these kernels need 10.0 (sm_100a, e.g. "
                "B200)",
                dev, d.major, d.minor);
  if (d.init_err != cudaSuccess)
    return fail(SVDQ_ERR_CUDA, "device setup: %s", cudaGetErrorString(d.init_err));
  unsigned long long id = current_ctx_id();
  if (id == 0 || id != d.ctx_id) {
    // first call in this context (the symbol lookup also makes the
    // device's primary context current if none was)
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_err_word);
    if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, "cudaGetSymbolAddress(error word): %s", cudaGetErrorString(e));
    id = current_ctx_id();
    if (id == 0) return fail(SVDQ_ERR_CUDA, "no current CUDA context on device %d", dev);
    d.err_word = static_cast<uint32_t*>(p);  // zero since the module loaded in this context
    d.attrs.clear();
    d.ctx_id = id;
  }
  ctx->stream = static_cast<cudaStream_t>(stream);
  ctx->device = dev;
  ctx->ctx_id = id;
  ctx->num_sms = d.num_sms;
  ctx->err_word = d.err_word;
  ctx->timeout_ns = g_timeout_ns;
  ctx->fault_flags = g_fault;
  ctx->gemm_pairs = g_gemm_pairs;
  ctx->pdl = g_pdl;
  return SVDQ_OK;
}

svdq_status ok() {
  t_detail[0] = '\0';
  return SVDQ_OK;
}

bool valid_rank(int r) { return r == 0 || r == 16 || r == 32 || r == 64 || r == 128; }

}  // namespace

svdq_status fail(svdq_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(t_detail, sizeof(t_detail), fmt, ap);
  va_end(ap);
  return st;
}

svdq_status set_smem_attr(const LaunchCtx& ctx, const void* kernel, int bytes) {
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[ctx.device];
  if (d.ctx_id != ctx.ctx_id) d.attrs.clear();  // another context since the call began
  for (const auto& a : d.attrs)
    if (a.first == kernel && a.second >= bytes) return SVDQ_OK;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(SVDQ_ERR_CUDA, "cudaFuncSetAttribute(%d bytes of shared memory): %s", bytes,
                cudaGetErrorString(e));
  }
  for (auto& a : d.attrs)
    if (a.first == kernel) {
      a.second = bytes;
      return SVDQ_OK;
    }
  d.attrs.emplace_back(kernel, bytes);
  return SVDQ_OK;
}

svdq_status check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return SVDQ_OK;
}

bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                  uint32_t elem_bytes, uint64_t rows, uint64_t cols, uint64_t row_stride_bytes,
                  uint32_t box_rows, uint32_t box_cols, int swizzle_bytes) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_NONE;
  if (swizzle_bytes == 128) sw = CU_TENSOR_MAP_SWIZZLE_128B;
  if (swizzle_bytes == 64) sw = CU_TENSOR_MAP_SWIZZLE_64B;
  if (swizzle_bytes == 32) sw = CU_TENSOR_MAP_SWIZZLE_32B;
  (void)elem_bytes;
  const CUresult r = g_encode(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) rows=%llu cols=%llu stride=%llu", (int)r,
         (unsigned long long)rows, (unsigned long long)cols, (unsigned long long)row_stride_bytes);
    return false;
  }
  return true;
}

bool make_tmap_3d_u8(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                     uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2, bool swizzle128) {
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {s1, s2};
  const cuuint32_t box[3] = {b0, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled (3-D) failed (%d) dims=%llu,%llu,%llu", (int)r,
         (unsigned long long)d0, (unsigned long long)d1, (unsigned long long)d2);
    return false;
  }
  return true;
}

}  // namespace svdq

using namespace svdq;

extern "C" {

int svdq_version(void) { return 100; }

const char* svdq_status_string(int status) {
  switch (status) {
    case SVDQ_OK: return "ok";
    case SVDQ_ERR_INVALID_ARG: return "invalid argument";
    case SVDQ_ERR_MISALIGNED: return "operand not 16-byte aligned";
    case SVDQ_ERR_UNSUPPORTED_DEVICE: return "unsupported device (needs compute capability 10.0, sm_100a)";
    case SVDQ_ERR_CUDA: return "CUDA error";
    case SVDQ_ERR_DEVICE_TIMEOUT: return "a bounded in-kernel wait timed out";
    case SVDQ_ERR_NOT_IMPLEMENTED: return "not implemented";
    default: return "unknown status";
  }
}

const char* svdq_last_error_detail(void) { return t_detail; }

size_t svdq_nvfp4_scale_bytes(int64_t rows, int64_t K) {
  if (rows <= 0 || K <= 0) return 0;
  const int64_t rp = (rows + 127) / 128 * 128;
  const int64_t cp = (K + 63) / 64 * 4;
  return static_cast<size_t>(rp * cp);
}

namespace {
svdq_status quantize_entry(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                              const float* smooth_s, const void* L1t_bf16, int r,
                              const float* act_gscale, float* act_gscale_out, uint8_t* q_out,
                              uint8_t* sf_out, float* lora_out, uint32_t* grid_sync, void* stream) {
  if (!x_bf16 || !q_out || !sf_out) return fail(SVDQ_ERR_INVALID_ARG, "x, q_out and sf_out must be non-null");
  if (M < 1 || M > (1ll << 30)) return fail(SVDQ_ERR_INVALID_ARG, "M=%lld out of range [1, 2^30]", (long long)M);
  if (K < 64 || K % 64 != 0 || K > (1ll << 20))
    return fail(SVDQ_ERR_INVALID_ARG, "K=%lld must be a positive multiple of 64 (<= 2^20)", (long long)K);
  if (ldx < K || ldx % 8 != 0)
    return fail(SVDQ_ERR_INVALID_ARG, "ldx=%lld must be >= K and a multiple of 8", (long long)ldx);
  if (!valid_rank(r)) return fail(SVDQ_ERR_INVALID_ARG, "rank r=%d must be 0, 16, 32, 64 or 128", r);
  if (r > 0 && (!L1t_bf16 || !lora_out))
    return fail(SVDQ_ERR_INVALID_ARG, "r > 0 needs L1t_bf16 and lora_out");
  if (!act_gscale && !act_gscale_out)
    return fail(SVDQ_ERR_INVALID_ARG, "dynamic scale (act_gscale == NULL) needs act_gscale_out");
  constexpr size_t kQuantSmemLimit = 227 * 1024 - 64;  // the opt-in limit less the static words
  if (quantize_smem_bytes(K, r) > kQuantSmemLimit) {
    int64_t kmax = K;  // the largest K this rank allows (error path only)
    while (kmax > 64 && quantize_smem_bytes(kmax, r) > kQuantSmemLimit) kmax -= 64;
    return fail(SVDQ_ERR_INVALID_ARG, "K=%lld with r=%d needs more than 227 KB of shared memory (K <= %lld at r=%d)",
                (long long)K, r, (long long)kmax, r);
  }
  if (!aligned16(x_bf16) || !aligned16(q_out) || !aligned16(sf_out) ||
      (r > 0 && (!aligned16(L1t_bf16) || !aligned16(lora_out))))
    return fail(SVDQ_ERR_MISALIGNED, "x, L1t, q_out, sf_out and lora_out must be 16-byte aligned");
  if ((smooth_s && (reinterpret_cast<uintptr_t>(smooth_s) & 3)) ||
      (act_gscale && (reinterpret_cast<uintptr_t>(act_gscale) & 3)) ||
      (act_gscale_out && (reinterpret_cast<uintptr_t>(act_gscale_out) & 3)))
    return fail(SVDQ_ERR_MISALIGNED, "fp32 operands must be 4-byte aligned");
  LaunchCtx ctx{};
  if (svdq_status e = device_ctx(stream, &ctx)) return e;
  if (svdq_status e = launch_quantize_act(ctx, x_bf16, M, K, ldx, smooth_s, L1t_bf16, r, act_gscale,
                                          act_gscale_out, q_out, sf_out, lora_out, grid_sync))
    return e;
  return ok();
}
}  // namespace

svdq_status svdq_quantize_act(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                              const float* smooth_s, const void* L1t_bf16, int r,
                              const float* act_gscale, float* act_gscale_out, uint8_t* q_out,
                              uint8_t* sf_out, float* lora_out, void* stream) {
  return quantize_entry(x_bf16, M, K, ldx, smooth_s, L1t_bf16, r, act_gscale, act_gscale_out, q_out,
                        sf_out, lora_out, nullptr, stream);
}

svdq_status svdq_quantize_act_dynamic(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                                      const float* smooth_s, const void* L1t_bf16, int r,
                                      float* act_gscale_out, void* workspace, uint8_t* q_out,
                                      uint8_t* sf_out, float* lora_out, void* stream) {
  if (!act_gscale_out || !workspace)
    return fail(SVDQ_ERR_INVALID_ARG, "act_gscale_out and workspace must be non-null");
  if (!aligned16(workspace)) return fail(SVDQ_ERR_MISALIGNED, "workspace must be 16-byte aligned");
  return quantize_entry(x_bf16, M, K, ldx, smooth_s, L1t_bf16, r, nullptr, act_gscale_out, q_out,
                        sf_out, lora_out, static_cast<uint32_t*>(workspace), stream);
}

svdq_status svdq_quantize_act_dynamic_noalloc(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                                              const float* smooth_s, const void* L1t_bf16, int r,
                                              float* act_gscale_out, uint8_t* q_out,
                                              uint8_t* sf_out, float* lora_out, void* stream) {
  if (!act_gscale_out) return fail(SVDQ_ERR_INVALID_ARG, "act_gscale_out must be non-null");
  LaunchCtx ctx{};
  if (svdq_status e = device_ctx(stream, &ctx)) return e;
  // the scratch this call needs (16 bytes) does not grow with M, K or r
  if (SVDQ_QUANTIZE_WORKSPACE_BYTES > kNoallocScratchBytes)
    return fail(SVDQ_ERR_INVALID_ARG, "scratch of %d bytes exceeds the %d-byte static array",
                SVDQ_QUANTIZE_WORKSPACE_BYTES, static_cast<int>(kNoallocScratchBytes));
  uint32_t* scratch = nullptr;
  if (svdq_status e = noalloc_quantize_scratch(ctx, &scratch)) return e;
  return quantize_entry(x_bf16, M, K, ldx, smooth_s, L1t_bf16, r, nullptr, act_gscale_out, q_out,
                        sf_out, lora_out, scratch, stream);
}

svdq_status svdq_w4a4_linear(const uint8_t* q_act, const uint8_t* sf_act, const float* act_gscale,
                             const float* lora_act, const uint8_t* q_w, const uint8_t* sf_w,
                             const float* w_gscale, const void* L2t_bf16, int r,
                             const void* bias_bf16, int64_t M, int64_t N, int64_t K, void* y_bf16,
                             int64_t ldy, void* stream) {
  return svdq_w4a4_linear_act(q_act, sf_act, act_gscale, lora_act, q_w, sf_w, w_gscale, L2t_bf16, r,
                              bias_bf16, M, N, K, y_bf16, ldy, SVDQ_ACT_NONE, stream);
}

svdq_status svdq_w4a4_linear_act(const uint8_t* q_act, const uint8_t* sf_act,
                                 const float* act_gscale, const float* lora_act, const uint8_t* q_w,
                                 const uint8_t* sf_w, const float* w_gscale, const void* L2t_bf16,
                                 int r, const void* bias_bf16, int64_t M, int64_t N, int64_t K,
                                 void* y_bf16, int64_t ldy, int activation, void* stream) {
  void* const parts[1] = {y_bf16};
  return svdq_w4a4_linear_split(q_act, sf_act, act_gscale, lora_act, q_w, sf_w, w_gscale, L2t_bf16,
                                r, bias_bf16, M, N, K, 1, parts, ldy, activation, stream);
}

svdq_status svdq_w4a4_linear_split(const uint8_t* q_act, const uint8_t* sf_act,
                                   const float* act_gscale, const float* lora_act,
                                   const uint8_t* q_w, const uint8_t* sf_w, const float* w_gscale,
                                   const void* L2t_bf16, int r, const void* bias_bf16, int64_t M,
                                   int64_t N, int64_t K, int parts, void* const* y_parts,
                                   int64_t ldy, int activation, void* stream) {
  if (activation != SVDQ_ACT_NONE && activation != SVDQ_ACT_GELU_TANH)
    return fail(SVDQ_ERR_INVALID_ARG, "activation=%d must be 0 (none) or 1 (GELU tanh)", activation);
  if (parts < 1 || parts > 3) return fail(SVDQ_ERR_INVALID_ARG, "parts=%d must be 1, 2 or 3", parts);
  if (!y_parts) return fail(SVDQ_ERR_INVALID_ARG, "y_parts must be non-null");
  for (int i = 0; i < parts; ++i)
    if (!y_parts[i]) return fail(SVDQ_ERR_INVALID_ARG, "y_parts[%d] must be non-null", i);
  if (!q_act || !sf_act || !act_gscale || !q_w || !sf_w || !w_gscale)
    return fail(SVDQ_ERR_INVALID_ARG, "q_act, sf_act, act_gscale, q_w, sf_w, w_gscale and y must be non-null");
  if (M < 1 || M > (1ll << 30)) return fail(SVDQ_ERR_INVALID_ARG, "M=%lld out of range [1, 2^30]", (long long)M);
  if (N < 16 || N % 16 != 0 || N > (1ll << 30))
    return fail(SVDQ_ERR_INVALID_ARG, "N=%lld must be a positive multiple of 16", (long long)N);
  if (parts > 1 && N % (128ll * parts) != 0)
    return fail(SVDQ_ERR_INVALID_ARG, "N=%lld: N/parts must be a multiple of 128 for parts=%d",
                (long long)N, parts);
  if (K < 64 || K % 64 != 0 || K > (1ll << 20))
    return fail(SVDQ_ERR_INVALID_ARG, "K=%lld must be a positive multiple of 64 (<= 2^20)", (long long)K);
  if (ldy < N / parts || ldy % 8 != 0)
    return fail(SVDQ_ERR_INVALID_ARG, "ldy=%lld must be >= N/parts and a multiple of 8", (long long)ldy);
  if (!valid_rank(r)) return fail(SVDQ_ERR_INVALID_ARG, "rank r=%d must be 0, 16, 32, 64 or 128", r);
  if (r > 0 && (!lora_act || !L2t_bf16)) return fail(SVDQ_ERR_INVALID_ARG, "r > 0 needs lora_act and L2t_bf16");
  bool ys_aligned = true;
  for (int i = 0; i < parts; ++i) ys_aligned = ys_aligned && aligned16(y_parts[i]);
  if (!aligned16(q_act) || !aligned16(sf_act) || !aligned16(q_w) || !aligned16(sf_w) ||
      !ys_aligned || (r > 0 && (!aligned16(L2t_bf16) || !aligned16(lora_act))))
    return fail(SVDQ_ERR_MISALIGNED, "codes, scales, lora_act, L2t and y must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(act_gscale) & 3) || (reinterpret_cast<uintptr_t>(w_gscale) & 3) ||
      (bias_bf16 && (reinterpret_cast<uintptr_t>(bias_bf16) & 1)))
    return fail(SVDQ_ERR_MISALIGNED, "scalars must be 4-byte and bias 2-byte aligned");
  LaunchCtx ctx{};
  if (svdq_status e = device_ctx(stream, &ctx)) return e;
  if (svdq_status e = launch_w4a4_gemm(ctx, q_act, sf_act, act_gscale, lora_act, q_w, sf_w, w_gscale,
                                       L2t_bf16, r, bias_bf16, M, N, K, parts, y_parts, ldy,
                                       activation))
    return e;
  return ok();
}

svdq_status awq_w4a16_linear(const void* x_bf16, int64_t M, int64_t K, const float* act_scale_inv,
                             const uint32_t* qweight, const void* scales_f16, const void* zeros_f16,
                             int group, const void* bias_bf16, int64_t N, void* y_bf16,
                             void* stream) {
  if (!x_bf16 || !qweight || !scales_f16 || !zeros_f16 || !y_bf16)
    return fail(SVDQ_ERR_INVALID_ARG, "x, qweight, scales, zeros and y must be non-null");
  if (M < 1 || M > 8) return fail(SVDQ_ERR_INVALID_ARG, "M=%lld must be in [1, 8]", (long long)M);
  if (group != 64) return fail(SVDQ_ERR_INVALID_ARG, "group=%d: only 64 is supported", group);
  const int64_t kmax = M <= 4 ? 14400 : 7104;  // B-fragment table must fit in 227 KB of smem
  if (K < 64 || K % 64 != 0 || K > kmax)
    return fail(SVDQ_ERR_INVALID_ARG, "K=%lld must be a multiple of 64 in [64, %lld] for M=%lld",
                (long long)K, (long long)kmax, (long long)M);
  if (N < 16 || N % 16 != 0 || N > (1ll << 30))
    return fail(SVDQ_ERR_INVALID_ARG, "N=%lld must be a positive multiple of 16", (long long)N);
  if (!aligned16(qweight) || !aligned16(x_bf16) || (act_scale_inv && !aligned16(act_scale_inv)))
    return fail(SVDQ_ERR_MISALIGNED, "x, act_scale_inv and qweight must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(y_bf16) & 1) || (reinterpret_cast<uintptr_t>(scales_f16) & 1) ||
      (reinterpret_cast<uintptr_t>(zeros_f16) & 1) ||
      (bias_bf16 && (reinterpret_cast<uintptr_t>(bias_bf16) & 1)))
    return fail(SVDQ_ERR_MISALIGNED, "y, scales, zeros and bias must be 2-byte aligned");
  LaunchCtx ctx{};
  if (svdq_status e = device_ctx(stream, &ctx)) return e;
  if (svdq_status e = launch_awq_w4a16(ctx, x_bf16, M, K, act_scale_inv, qweight, scales_f16,
                                       zeros_f16, bias_bf16, N, y_bf16))
    return e;
  return ok();
}

svdq_status svdq_check_device_errors(void* stream) {
  LaunchCtx ctx{};
  if (svdq_status e = device_ctx(stream, &ctx)) return e;
  cudaError_t e = cudaStreamSynchronize(ctx.stream);
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, "stream: %s", cudaGetErrorString(e));
  uint32_t word = 0;
  e = cudaMemcpy(&word, ctx.err_word, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, "reading the error word: %s", cudaGetErrorString(e));
  if (word) {
    cudaMemset(ctx.err_word, 0, sizeof(uint32_t));
    return fail(SVDQ_ERR_DEVICE_TIMEOUT, "device error word 0x%x (1 data wait, 2 slot wait, 4 "
                "accumulator wait, 8 drain, 16 grid barrier)", word);
  }
  return ok();
}

uint64_t svdq_set_wait_timeout_ns(uint64_t ns) {
  std::lock_guard<std::mutex> lk(g_mu);
  const uint64_t prev = g_timeout_ns;
  g_timeout_ns = ns ? ns : 2000000000ull;
  return prev;
}

int svdq_set_gemm_pairs(int enable) {
  std::lock_guard<std::mutex> lk(g_mu);
  const int prev = g_gemm_pairs;
  g_gemm_pairs = enable ? 1 : 0;
  return prev;
}

int svdq_set_pdl(int enable) {
  std::lock_guard<std::mutex> lk(g_mu);
  const int prev = g_pdl;
  g_pdl = enable ? 1 : 0;
  return prev;
}

int svdq_debug_set_fault(int flags) {
  std::lock_guard<std::mutex> lk(g_mu);
  const int prev = g_fault;
  g_fault = flags;
  return prev;
}

}  // extern "C"
