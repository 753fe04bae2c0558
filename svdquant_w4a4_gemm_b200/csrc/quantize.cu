// quantize.cu — svdq_quantize_act: smoothing, NVFP4 activation quantization
// and the low-rank down-projection in one pass over x.
//
// The pages fuse the low-rank down-projection with the quantization kernel
// so that the 16-bit branch costs no extra pass over the activations
// ("Bringing Nunchaku 4-bit Diffusion Inference to Diffusers", as told on
// blog.margrop.com "技术细节 §1", SVDQuant step 4).
//
// Work unit: a 128-row x 64-column sub-tile of x (16 KB of bf16, one
// 128-byte-swizzled TMA box).  The ceil(M/128)·(K/64) sub-tiles, in
// row-block-major order, are split into one contiguous, equal range per CTA
// (one persistent CTA per SM), so the memory pipeline never drains between
// work items and the load is balanced to one sub-tile.
//   warp 0       TMA producer: x sub-tiles and the matching 64-column slices
//                of L1ᵀ into a kStages-deep shared-memory ring; its lanes
//                also compute RN(1/s) for the slot's 64 columns.
//   warp 1       TMEM owner; one thread issues the down-projection as
//                tcgen05 kind::f16 MMAs (M = 128, N = r, K = 16 each) from
//                the quantized tile's bf16(x̂) and the L1ᵀ slice into a TMEM
//                accumulator; a new accumulator (of two) per run of
//                sub-tiles in the same 128-row block ("segment").
//   warps 2-9    quantizers: one thread = one row x 32 columns = two
//                16-element groups: x̂ = x·inv_s, group max, E4M3 scale
//                (cvt.rn.satfinite.e4m3x2), E2M1 codes (cvt.rn.satfinite
//                .e2m1x2, sign bit copied), a 16-byte code store, a 2-byte
//                scale store into the 128x4 block layout, and bf16(x̂)
//                written back over the tile for the MMA.
//   warps 10-13  epilogue: when a segment's accumulator is complete, TMEM ->
//                registers -> float4 atomics into xl (zeroed beforehand:
//                a row block's K range can span several CTAs), then release
//                the accumulator.
// HBM traffic is the algorithmic minimum: x once, codes + scales + xl once;
// L1ᵀ slices come from L2.
#include <cstdio>

#include "internal.h"
#include "ptx.cuh"

namespace svdq {
namespace {

constexpr int kBM = 128;
constexpr int kSubK = 64;
constexpr int kStages = 4;
constexpr int kQuantWarps = 8;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 32 * (2 + kQuantWarps + kEpiWarps);
constexpr uint32_t kXTileBytes = kBM * kSubK * 2;

struct QuantParams {
  int M, K, r;
  int units;              // ceil(M/128) * (K/64) sub-tiles
  const float* smooth_s;  // [K] or null
  const float* gs_in;     // static tensor scale, or null for dynamic
  const float* amax_src;  // dynamic: amax bits (written by the amax pass)
  float* gs_copy;         // static: where to copy gs (block 0), or null
  uint8_t* q_out;
  uint8_t* sf_out;
  float* lora_out;
  WaitCfg wait;
};

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Copy each value's sign into bit 3 of its nibble (a value that rounds to
// zero keeps its sign: E2M1 code 0x8 for negative inputs).
__device__ __forceinline__ uint32_t e2m1_signs(const float (&v)[8]) {
  uint32_t s = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) s |= (__float_as_uint(v[i]) >> 31) << (4 * i + 3);
  return s;
}

__device__ __forceinline__ float tensor_scale_from_amax(float amax) {
  return amax > 0.0f ? __fdiv_rn(2688.0f, amax) : 1.0f;
}

// This CTA's contiguous range of sub-tiles.
__device__ __forceinline__ void unit_range(int units, int& u0, int& u1) {
  u0 = static_cast<int>((static_cast<int64_t>(blockIdx.x) * units) / gridDim.x);
  u1 = static_cast<int>((static_cast<int64_t>(blockIdx.x + 1) * units) / gridDim.x);
}

__global__ void __launch_bounds__(kThreads, 1)
    quantize_act_kernel(const __grid_constant__ CUtensorMap tmap_x,
                        const __grid_constant__ CUtensorMap tmap_l1, const QuantParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t l1_bytes = static_cast<uint32_t>(p.r) * 128u;
  uint8_t* xs = base;
  uint8_t* ls = xs + kStages * kXTileBytes;
  float* inv_st = reinterpret_cast<float*>(ls + kStages * l1_bytes);  // [kStages][64]
  uint64_t* full = reinterpret_cast<uint64_t*>(inv_st + kStages * kSubK);
  uint64_t* qdone = full + kStages;
  uint64_t* empty = qdone + kStages;
  uint64_t* acc_full = empty + kStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kblocks = p.K / kSubK;
  const bool has_lr = p.r > 0;
  const uint32_t tmem_cols = p.r <= 16 ? 32u : static_cast<uint32_t>(2 * p.r);
  int u0, u1;
  unit_range(p.units, u0, u1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&qdone[s], kQuantWarps);
      mbar_init(&empty[s], has_lr ? 1 : kQuantWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
    }
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_x);
    if (has_lr) tma_prefetch_desc(&tmap_l1);
  }
  if (warp == 1 && has_lr) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = has_lr ? *tmem_slot : 0u;

  if (warp == 0) {
    // ------------------------------------------------------- producer ----
    int issued = 0;
    for (int u = u0; u < u1; ++u) {
      const int i = u - u0;
      const int s = i % kStages;
      const uint32_t ph = (i / kStages) & 1;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&empty[s], ph ^ 1, p.wait, kErrTimeoutEmpty) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      const int rb = u / kblocks, kb = u % kblocks;
      // RN(1/s) of this slot's 64 columns, published by the arrive below
      float2 iv = make_float2(1.0f, 1.0f);
      if (p.smooth_s) {
        const float2 sv = *reinterpret_cast<const float2*>(p.smooth_s + kb * kSubK + 2 * lane);
        iv = make_float2(__fdiv_rn(1.0f, sv.x), __fdiv_rn(1.0f, sv.y));
      }
      reinterpret_cast<float2*>(inv_st + s * kSubK)[lane] = iv;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], kXTileBytes + (has_lr ? l1_bytes : 0u));
        tma_load_2d(xs + s * kXTileBytes, &tmap_x, &full[s], kb * kSubK, rb * kBM);
        if (has_lr) tma_load_2d(ls + s * l1_bytes, &tmap_l1, &full[s], kb * kSubK, 0);
      }
      issued = i + 1;
    }
    // never leave the CTA with a copy still landing in its shared memory
    if (lane == 0)
      for (int i = max(0, issued - kStages); i < issued; ++i)
        mbar_wait(&full[i % kStages], (i / kStages) & 1, p.wait, kErrTimeoutDrain);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA ----
    if (has_lr && lane == 0) {
      const uint32_t idesc = idesc_f16(128, static_cast<uint32_t>(p.r), true);
      int seg = 0;             // segments started by this CTA
      bool first = true;       // first sub-tile of the current segment
      for (int u = u0; u < u1; ++u) {
        const int i = u - u0;
        const int s = i % kStages;
        const uint32_t ph = (i / kStages) & 1;
        const int buf = seg & 1;
        if (first && seg >= 2 &&
            !mbar_wait(&acc_empty[buf], ((seg >> 1) - 1) & 1, p.wait, kErrTimeoutAcc))
          break;
        if (!mbar_wait(&qdone[s], ph, p.wait, kErrTimeoutFull)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(xs + s * kXTileBytes);
        const uint32_t b0 = smem_u32(ls + s * l1_bytes);
        const uint32_t d = tmem + buf * static_cast<uint32_t>(p.r);
#pragma unroll
        for (int kk = 0; kk < kSubK / 16; ++kk) {
          const uint64_t ad = make_sdesc(a0 + kk * 32, 16, 1024, kSwz128);
          const uint64_t bd = make_sdesc(b0 + kk * 32, 16, 1024, kSwz128);
          umma_f16(d, ad, bd, idesc, (!first || kk > 0) ? 1u : 0u);
        }
        umma_commit(&empty[s]);
        first = false;
        const bool seg_end = (u + 1 == u1) || ((u + 1) / kblocks != u / kblocks);
        if (seg_end) {
          umma_commit(&acc_full[buf]);
          ++seg;
          first = true;
        }
      }
    }
  } else if (warp < 2 + kQuantWarps) {
    // ------------------------------------------------------ quantizers ----
    const int qw = warp - 2;
    const int row = 32 * (qw & 3) + lane;  // row within the tile
    const int half = qw >> 2;              // which 32 of the 64 columns
    float gs;
    if (p.gs_in) {
      gs = *p.gs_in;
    } else {
      gs = tensor_scale_from_amax(*p.amax_src);
    }
    if (p.gs_copy && blockIdx.x == 0 && threadIdx.x == 64) *p.gs_copy = gs;
    const size_t kbytes = static_cast<size_t>(p.K) / 2;
    for (int u = u0; u < u1; ++u) {
      const int i = u - u0;
      const int s = i % kStages;
      const uint32_t ph = (i / kStages) & 1;
      if (!mbar_wait(&full[s], ph, p.wait, kErrTimeoutFull)) break;
      const int rb = u / kblocks, kb = u % kblocks;
      const int grow = rb * kBM + row;
      uint8_t* trow = xs + s * kXTileBytes + row * 128;
      const int kc0 = kb * kSubK + 32 * half;  // first column of this thread
      const float* inv_s = inv_st + s * kSubK + 32 * half;
      uint4 v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        v[j] = *reinterpret_cast<const uint4*>(trow + (((4 * half + j) ^ (row & 7)) << 4));
      uint32_t codes[4];
      uint32_t sfb[2];
      uint4 back[4];
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const uint32_t w[8] = {v[2 * g].x,     v[2 * g].y,     v[2 * g].z,     v[2 * g].w,
                               v[2 * g + 1].x, v[2 * g + 1].y, v[2 * g + 1].z, v[2 * g + 1].w};
        float xh[16];
        const float4* is4 = reinterpret_cast<const float4*>(inv_s + 16 * g);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 iv = is4[q];
          xh[4 * q + 0] = __fmul_rn(bf16lo(w[2 * q]), iv.x);
          xh[4 * q + 1] = __fmul_rn(bf16hi(w[2 * q]), iv.y);
          xh[4 * q + 2] = __fmul_rn(bf16lo(w[2 * q + 1]), iv.z);
          xh[4 * q + 3] = __fmul_rn(bf16hi(w[2 * q + 1]), iv.w);
        }
        float amax = 0.0f;
#pragma unroll
        for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(xh[e]));
        const float t = __fmul_rn(__fdiv_rn(amax, 6.0f), gs);
        const uint32_t sf = cvt_e4m3(t);
        const float d = e4m3_to_f32(sf);
        const float inv = d == 0.0f ? 0.0f : __fdiv_rn(gs, d);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float q8[8], x8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            x8[e] = xh[8 * h + e];
            q8[e] = __fmul_rn(x8[e], inv);
          }
          codes[2 * g + h] = cvt_e2m1x8(q8) | e2m1_signs(x8);
        }
        sfb[g] = sf;
        if (has_lr) {
#pragma unroll
          for (int h = 0; h < 2; ++h)
            back[2 * g + h] = make_uint4(pack_bf16x2(xh[8 * h + 0], xh[8 * h + 1]),
                                         pack_bf16x2(xh[8 * h + 2], xh[8 * h + 3]),
                                         pack_bf16x2(xh[8 * h + 4], xh[8 * h + 5]),
                                         pack_bf16x2(xh[8 * h + 6], xh[8 * h + 7]));
        }
      }
      if (grow < p.M) {
        *reinterpret_cast<uint4*>(p.q_out + static_cast<size_t>(grow) * kbytes + kc0 / 2) =
            make_uint4(codes[0], codes[1], codes[2], codes[3]);
      }
      // rows past M inside the last 128-row block hold zero-filled x, so
      // their scales are written as the zero padding the layout requires
      *reinterpret_cast<uint16_t*>(p.sf_out + (static_cast<size_t>(rb) * kblocks + kb) * 512 +
                                   (row & 31) * 16 + (row >> 5) * 4 + 2 * half) =
          static_cast<uint16_t>(sfb[0] | (sfb[1] << 8));
      if (has_lr) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<uint4*>(trow + (((4 * half + j) ^ (row & 7)) << 4)) = back[j];
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&qdone[s]);
      } else {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
    }
  } else {
    // ------------------------------------------------- xl epilogue ----
    if (has_lr) {
      const int quad = warp & 3;
      int seg = 0;
      for (int u = u0; u < u1; ++u) {
        const bool seg_end = (u + 1 == u1) || ((u + 1) / kblocks != u / kblocks);
        if (!seg_end) continue;
        const int buf = seg & 1;
        if (!mbar_wait(&acc_full[buf], (seg >> 1) & 1, p.wait, kErrTimeoutAcc)) break;
        tc_fence_after();
        const int grow = (u / kblocks) * kBM + 32 * quad + lane;
        const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * quad) << 16) + buf * p.r;
        for (int c = 0; c < p.r / 16; ++c) {
          uint32_t acc[16];
          tmem_ld_32x32b_x16(taddr + c * 16, acc);
          tmem_ld_wait();
          if (grow < p.M) {
            float4* dst = reinterpret_cast<float4*>(p.lora_out + static_cast<size_t>(grow) * p.r + c * 16);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              atomicAdd(dst + q, make_float4(__uint_as_float(acc[4 * q]), __uint_as_float(acc[4 * q + 1]),
                                             __uint_as_float(acc[4 * q + 2]),
                                             __uint_as_float(acc[4 * q + 3])));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
        ++seg;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1 && has_lr) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

// Dynamic tensor scale, pass 1: max|x·inv_s| over the tensor into *amax_bits
// (non-negative floats order like their bit patterns, so atomicMax works).
__global__ void __launch_bounds__(256) act_amax_kernel(const uint16_t* __restrict__ x, int M, int K,
                                                       int64_t ldx, const float* __restrict__ s,
                                                       unsigned* amax_bits) {
  const int c8 = blockIdx.x * blockDim.x + threadIdx.x;  // which 8-column chunk
  float m = 0.0f;
  if (c8 * 8 < K) {
    float inv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) inv[e] = s ? __fdiv_rn(1.0f, s[c8 * 8 + e]) : 1.0f;
    for (int row = blockIdx.y; row < M; row += gridDim.y) {
      const uint4 v = *reinterpret_cast<const uint4*>(x + row * ldx + c8 * 8);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        m = fmaxf(m, fabsf(__fmul_rn(bf16lo(w[q]), inv[2 * q])));
        m = fmaxf(m, fabsf(__fmul_rn(bf16hi(w[q]), inv[2 * q + 1])));
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wm[8];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i) m = fmaxf(m, wm[i]);
    atomicMax(amax_bits, __float_as_uint(m));
  }
}

// Dynamic tensor scale, pass 3: turn the amax bits into gs in place.
__global__ void act_scale_finalize_kernel(float* gs) {
  const float amax = __uint_as_float(*reinterpret_cast<unsigned*>(gs));
  *gs = tensor_scale_from_amax(amax);
}

}  // namespace

svdq_status launch_quantize_act(const LaunchCtx& ctx, const void* x, int64_t M, int64_t K,
                                int64_t ldx, const float* smooth_s, const void* L1t, int r,
                                const float* act_gscale, float* act_gscale_out, uint8_t* q_out,
                                uint8_t* sf_out, float* lora_out) {
  if (smooth_s && (reinterpret_cast<uintptr_t>(smooth_s) & 7))
    return fail(SVDQ_ERR_MISALIGNED, "smooth_s must be 8-byte aligned");
  CUtensorMap tx{}, tl{};
  if (!make_tmap_2d(&tx, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, K, ldx * 2, kBM, kSubK, 128))
    return SVDQ_ERR_CUDA;
  if (r > 0 && !make_tmap_2d(&tl, L1t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, r, K, K * 2, r,
                             kSubK, 128))
    return SVDQ_ERR_CUDA;
  if (r == 0) tl = tx;

  QuantParams p{};
  p.M = static_cast<int>(M);
  p.K = static_cast<int>(K);
  p.r = r;
  p.units = static_cast<int>(((M + kBM - 1) / kBM) * (K / kSubK));
  p.smooth_s = smooth_s;
  p.gs_in = act_gscale;
  p.amax_src = act_gscale ? nullptr : act_gscale_out;
  p.gs_copy = (act_gscale && act_gscale_out && act_gscale_out != act_gscale) ? act_gscale_out
                                                                              : nullptr;
  p.q_out = q_out;
  p.sf_out = sf_out;
  p.lora_out = lora_out;
  p.wait = WaitCfg{ctx.timeout_ns, ctx.err_word};

  cudaStream_t st = ctx.stream;
  if (r > 0 && cudaMemsetAsync(lora_out, 0, static_cast<size_t>(M) * r * 4, st) != cudaSuccess)
    return check_launch("memset lora_out");
  if (!act_gscale) {
    if (cudaMemsetAsync(act_gscale_out, 0, 4, st) != cudaSuccess) return check_launch("memset gs");
    const int bx = static_cast<int>((K / 8 + 255) / 256);
    const int by = static_cast<int>(std::min<int64_t>(M, std::max(1, 4 * ctx.num_sms / bx)));
    act_amax_kernel<<<dim3(bx, by), 256, 0, st>>>(static_cast<const uint16_t*>(x), p.M, p.K, ldx,
                                                  smooth_s, reinterpret_cast<unsigned*>(act_gscale_out));
    if (svdq_status e = check_launch("act_amax_kernel")) return e;
  }
  const size_t smem = 1024 + kStages * (kXTileBytes + static_cast<size_t>(r) * 128 + kSubK * 4) +
                      8 * (3 * kStages + 4) + 16;
  static bool attr_done[64] = {};
  if (!attr_done[ctx.device & 63]) {
    cudaFuncSetAttribute(quantize_act_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         227 * 1024);
    attr_done[ctx.device & 63] = true;
  }
  const int grid = std::min(p.units, ctx.num_sms);
  quantize_act_kernel<<<grid, kThreads, smem, st>>>(tx, tl, p);
  if (svdq_status e = check_launch("quantize_act_kernel")) return e;
  if (!act_gscale) {
    act_scale_finalize_kernel<<<1, 1, 0, st>>>(act_gscale_out);
    if (svdq_status e = check_launch("act_scale_finalize_kernel")) return e;
  }
  return SVDQ_OK;
}

}  // namespace svdq
