// internal.h — host-side plumbing shared by the library's translation units.
#pragma once

#include <utility>

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "svdq.h"

namespace svdq {

// Per-launch context the API layer fills in after validation.
struct LaunchCtx {
  cudaStream_t stream;
  int device;
  unsigned long long ctx_id;  // current CUDA context (its process-unique ID)
  int num_sms;
  uint32_t* err_word;    // device error word of `device`
  uint64_t timeout_ns;   // bound on every in-kernel wait
  int fault_flags;       // test-only fault injection
  int gemm_pairs;        // 1: W4A4 GEMM on SM pairs where the shape allows (svdq_set_gemm_pairs)
  int pdl;               // 1: launches may overlap the previous kernel's tail (svdq_set_pdl)
};

// Encode a 2-D tiled tensor map (row-major [rows, cols] of `elem_bytes`
// elements, row stride `row_stride_bytes`), box [box_rows, box_cols].
// swizzle_bytes: 0, 32, 64 or 128.  Returns false and sets the detail on error.
bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                  uint32_t elem_bytes, uint64_t rows, uint64_t cols, uint64_t row_stride_bytes,
                  uint32_t box_rows, uint32_t box_cols, int swizzle_bytes);

// A 3-D tiled tensor map over bytes: dims (d0, d1, d2) with byte strides s1
// (between d1 indices) and s2 (between d2 indices), box (b0, b1, b2), 128-byte
// swizzle when swizzle128.  Returns false and sets the detail on error.
bool make_tmap_3d_u8(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                     uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2, bool swizzle128);

// Thread-local error detail (api.cu).
svdq_status fail(svdq_status st, const char* fmt, ...);
svdq_status check_launch(const char* what);

// Launches kern<<<grid, block, smem, ctx.stream>>>(args...) through
// cudaLaunchKernelEx, with programmatic dependent launch allowed when
// ctx.pdl: the kernel may then be scheduled while the previous kernel on the
// stream is still finishing.  Every kernel of this library waits for its
// predecessor (griddepcontrol.wait) before its first global memory access,
// so stream order holds for every operand; what overlaps is the launch and
// the set-up (barrier initialisation, tensor memory allocation, descriptor
// prefetch).  A kernel compiled with __cluster_dims__ keeps its clusters.
template <typename... KArgs, typename... Args>
svdq_status launch_kernel(const LaunchCtx& ctx, const char* what, void (*kern)(KArgs...), dim3 grid,
                          dim3 block, size_t smem, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = ctx.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = ctx.pdl ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return check_launch(what);
}

// Opt `kernel` in to `bytes` of dynamic shared memory in the current context
// (once per context and kernel; thread-safe).  SVDQ_ERR_CUDA if refused.
svdq_status set_smem_attr(const LaunchCtx& ctx, const void* kernel, int bytes);

// Shared memory the quantize kernel needs for a [*, K] activation at rank r
// (the API rejects shapes above the 227 KB per-CTA limit before launching).
size_t quantize_smem_bytes(int64_t K, int r);

// Bytes of the static scratch array behind svdq_quantize_act_dynamic_noalloc,
// and its device address in the current context of ctx.device.
constexpr size_t kNoallocScratchBytes = 256;
svdq_status noalloc_quantize_scratch(const LaunchCtx& ctx, uint32_t** out);

// Kernel launchers (one per translation unit).  Arguments are validated.
svdq_status launch_quantize_act(const LaunchCtx& ctx, const void* x, int64_t M, int64_t K,
                                int64_t ldx, const float* smooth_s, const void* L1t, int r,
                                const float* act_gscale, float* act_gscale_out, uint8_t* q_out,
                                uint8_t* sf_out, float* lora_out, uint32_t* grid_sync = nullptr);

svdq_status launch_w4a4_gemm(const LaunchCtx& ctx, const uint8_t* q_act, const uint8_t* sf_act,
                             const float* act_gscale, const float* lora_act, const uint8_t* q_w,
                             const uint8_t* sf_w, const float* w_gscale, const void* L2t, int r,
                             const void* bias, int64_t M, int64_t N, int64_t K, int parts,
                             void* const* y_parts, int64_t ldy, int activation);

svdq_status launch_awq_w4a16(const LaunchCtx& ctx, const void* x, int64_t M, int64_t K,
                             const float* act_scale_inv, const uint32_t* qweight,
                             const void* scales, const void* zeros, const void* bias, int64_t N,
                             void* y);

}  // namespace svdq
