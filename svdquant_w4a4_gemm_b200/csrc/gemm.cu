// gemm.cu — svdq_w4a4_linear: the NVFP4 W4A4 GEMM with the low-rank
// up-projection fused in ("the low-rank up-projection is fused with the
// 4-bit compute kernel", blog.margrop.com "技术细节 §1", SVDQuant step 4).
//
//   y = bf16( α·acc + bias ),  α = 1/(gs_a·gs_w)
//   acc = (hi + lo)·L2                      (kind::f16 MMAs, first)
//       + Σ_k e2m1_a·sfa · e2m1_w·sfw      (kind::mxf4nvf4 block-scaled MMAs)
//   hi = bf16(xl·gs_a·gs_w), lo = bf16(xl·gs_a·gs_w − hi)
// The low-rank term can dominate y (it carries the outlier channels), so
// its activation operand keeps ~16 significant bits through the hi/lo
// split; L2 itself is bf16 by construction.
//
// One CTA computes a 128 x BN tile of y (BN = 256, or 128 when N is not a
// multiple of 256), fp32 accumulator in tensor memory (TMEM).
//   warp 0     producer: TMA loads of the packed FP4 operands (128-byte rows,
//              128-byte swizzle: 16 KB of A and BN x 128 B of B per stage,
//              256 K-elements), plain bulk copies of the matching scale
//              blocks (the 128x4 block layout is already the byte order the
//              scale copy to TMEM wants: 2 KB per 128 rows per stage), and
//              TMA loads of L2ᵀ for the low-rank steps.
//   warp 1     TMEM owner and MMA issuer (one thread): per stage it copies
//              the stage's scale blocks smem -> TMEM (tcgen05.cp 32x128b
//              .warpx4, 4 columns per 128 rows per 64 K) and issues four
//              block-scaled MMAs (K = 64 each); tcgen05.commit frees the stage.
//   warps 2-5  first convert the [128 x r] fp32 down-projection rows into
//              the hi/lo bf16 parts in the A slot of the first ring stages
//              (128-byte swizzle written by hand), then run the epilogue:
//              TMEM -> registers, α·acc + bias, bf16, store.
// The low-rank steps go through the same shared-memory ring as the FP4
// stages, so they need no memory of their own: for r <= 32 one ring slot
// holds hi in A columns [0, 32) and lo in [32, 64) against one L2ᵀ slice;
// for r = 64, 128 each 64-wide slice of r takes two slots (hi, then lo),
// both loading the same L2ᵀ slice.
#include "internal.h"
#include "ptx.cuh"

namespace svdq {
namespace {

constexpr int kBM = 128;
constexpr int kBKBytes = 128;  // 256 FP4 elements per stage and row
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr uint32_t kATileBytes = kBM * kBKBytes;  // 16 KB

struct GemmParams {
  int M, N, K, r, bn;
  const uint8_t* sf_a;
  const uint8_t* sf_w;
  const float* gs_a;
  const float* gs_w;
  const float* lora;      // [M, r]
  const uint16_t* bias;   // [N] or null
  uint16_t* y;
  int64_t ldy;
  int fault;              // test hook: 1 = skip the first stage's loads
  WaitCfg wait;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int BN>
struct Layout {
  static constexpr uint32_t kB = BN * kBKBytes;          // B tile bytes
  static constexpr uint32_t kSfa = 4 * 512;              // 4 K-blocks x 128 rows
  static constexpr uint32_t kSfb = (BN / 128) * 4 * 512;
  static constexpr uint32_t kStage = kATileBytes + kB + kSfa + kSfb;
  static constexpr uint32_t kTmemCols = 512;             // acc BN + scales
  static constexpr uint32_t kSfaCol = BN;                // 16 columns
  static constexpr uint32_t kSfbCol = BN + 16;           // (BN/128)*16 columns
  static_assert(kStage % 1024 == 0, "stage must keep 1 KB alignment");
  static_assert(BN + 16 + (BN / 128) * 16 <= 512, "TMEM budget");
};

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                     const __grid_constant__ CUtensorMap tmap_b,
                     const __grid_constant__ CUtensorMap tmap_l2, const GemmParams p) {
  using L = Layout<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kStages * L::kStage);
  uint64_t* empty = full + kStages;
  uint64_t* lr_full = empty + kStages;
  uint64_t* acc_full = lr_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  auto stage_a = [&](int s) { return base + s * L::kStage; };
  auto stage_b = [&](int s) { return base + s * L::kStage + kATileBytes; };
  auto stage_sfa = [&](int s) { return base + s * L::kStage + kATileBytes + L::kB; };
  auto stage_sfb = [&](int s) { return base + s * L::kStage + kATileBytes + L::kB + L::kSfa; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN;
  const int m0 = blockIdx.y * kBM;
  const bool lr_packed = p.r > 0 && p.r <= 32;  // hi and lo share one A tile
  const int nlr = p.r == 0 ? 0 : (lr_packed ? 1 : 2 * (p.r / 64));  // low-rank ring steps
  const int kblocks = p.K / 64;              // 64-element K blocks (one MMA each)
  const int nk = (kblocks + 3) / 4;          // FP4 ring steps (256 K each, last may be short)
  const int nsteps = nlr + nk;
  const int nb_total = (p.N + 127) / 128;    // 128-row blocks of the weight scales

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(lr_full, 4);
    mbar_init(acc_full, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b);
    if (p.r > 0) tma_prefetch_desc(&tmap_l2);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------- producer ----
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % kStages;
        const uint32_t ph = (i / kStages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, p.wait, kErrTimeoutEmpty)) break;
        if (p.fault == 1 && i == 0) continue;  // test hook: this stage never fills
        if (i < nlr) {
          // L2ᵀ[n0 .. n0+BN) x r[64c .. 64c+64) as bf16, zero-filled past r
          const int c = lr_packed ? 0 : i / 2;
          mbar_arrive_expect_tx(&full[s], L::kB);
          tma_load_2d(stage_b(s), &tmap_l2, &full[s], 64 * c, n0);
        } else {
          const int kb = i - nlr;  // 256-element K step
          const int nkb = min(4, kblocks - 4 * kb);                  // scale blocks (MMAs) in it
          const int nbl = min(BN / 128, nb_total - n0 / 128);        // weight scale row blocks
          const uint32_t sfbytes = static_cast<uint32_t>(nkb) * 512;
          mbar_arrive_expect_tx(&full[s], kATileBytes + L::kB + sfbytes * (1 + nbl));
          tma_load_2d(stage_a(s), &tmap_a, &full[s], kb * kBKBytes, m0);
          tma_load_2d(stage_b(s), &tmap_b, &full[s], kb * kBKBytes, n0);
          bulk_load(stage_sfa(s), p.sf_a + (static_cast<size_t>(m0 / 128) * kblocks + 4 * kb) * 512,
                    sfbytes, &full[s]);
          for (int nb = 0; nb < nbl; ++nb)
            bulk_load(stage_sfb(s) + nb * 2048,
                      p.sf_w + (static_cast<size_t>(n0 / 128 + nb) * kblocks + 4 * kb) * 512,
                      sfbytes, &full[s]);
        }
        issued = i + 1;
      }
      for (int i = max(0, issued - kStages); i < issued; ++i) {
        if (p.fault == 1 && i == 0) continue;
        mbar_wait(&full[i % kStages], (i / kStages) & 1, p.wait, kErrTimeoutDrain);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA ----
    if (lane == 0) {
      const uint32_t id_f16 = idesc_f16(128, BN, true);
      const uint32_t id_fp4 = idesc_nvfp4(128, BN);
      bool ok = true;
      if (nlr > 0 && !mbar_wait(lr_full, 0, p.wait, kErrTimeoutFull)) ok = false;
      tc_fence_after();
      for (int i = 0; ok && i < nsteps; ++i) {
        const int s = i % kStages;
        const uint32_t ph = (i / kStages) & 1;
        if (!mbar_wait(&full[s], ph, p.wait, kErrTimeoutFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(stage_a(s));
        const uint32_t b0 = smem_u32(stage_b(s));
        if (i < nlr) {
          // packed: A k-steps [0, r/16) hold hi and [2, 2 + r/16) hold lo,
          // both against B k-steps [0, r/16); unpacked: 4 k-steps per slot
          const int ksteps = lr_packed ? p.r / 16 : 4;
          for (int kk = 0; kk < ksteps; ++kk) {
            const uint64_t bd = make_sdesc(b0 + kk * 32, 16, 1024, kSwz128);
            umma_f16(tmem, make_sdesc(a0 + kk * 32, 16, 1024, kSwz128), bd, id_f16,
                     (i > 0 || kk > 0) ? 1u : 0u);
            if (lr_packed)
              umma_f16(tmem, make_sdesc(a0 + (2 + kk) * 32, 16, 1024, kSwz128), bd, id_f16, 1u);
          }
        } else {
          const uint32_t sa = smem_u32(stage_sfa(s));
          const uint32_t sb = smem_u32(stage_sfb(s));
          const int nkb = min(4, kblocks - 4 * (i - nlr));
          for (int kk = 0; kk < nkb; ++kk) {
            tmem_cp_32x128b_warpx4(tmem + L::kSfaCol + 4 * kk, make_sdesc(sa + kk * 512, 128, 128, kSwzNone));
#pragma unroll
            for (int nb = 0; nb < BN / 128; ++nb)
              tmem_cp_32x128b_warpx4(tmem + L::kSfbCol + (BN / 128) * 4 * kk + 4 * nb,
                                     make_sdesc(sb + (nb * 4 + kk) * 512, 128, 128, kSwzNone));
          }
          for (int kk = 0; kk < nkb; ++kk) {
            const uint64_t ad = make_sdesc(a0 + kk * 32, 16, 1024, kSwz128);
            const uint64_t bd = make_sdesc(b0 + kk * 32, 16, 1024, kSwz128);
            umma_nvfp4(tmem, ad, bd, id_fp4, tmem + L::kSfaCol + 4 * kk,
                       tmem + L::kSfbCol + (BN / 128) * 4 * kk,
                       (i > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&empty[s]);
      }
      if (ok) umma_commit(acc_full);
    }
  } else {
    // --------------------------------------- low-rank A, then epilogue ----
    const int quad = warp & 3;
    const int row = 32 * quad + lane;  // TMEM lane == tile row
    const int grow = m0 + row;
    const float gsa = *p.gs_a, gsw = *p.gs_w;
    const float gprod = __fmul_rn(gsa, gsw);
    const float alpha = __fdiv_rn(1.0f, gprod);
    if (nlr > 0) {
      // this row's xl·gs_a·gs_w split into bf16 hi + lo parts
      for (int step = 0; step < nlr; ++step) {
        uint8_t* arow = stage_a(step % kStages) + row * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {  // 8 bf16 = one 16-byte chunk
          // packed: chunks 0-3 = hi of columns 0..31, chunks 4-7 = lo of them;
          // unpacked: slice step/2, part step%2 (0 = hi, 1 = lo)
          const int part = lr_packed ? (j >> 2) : (step & 1);
          const int col0 = lr_packed ? 8 * (j & 3) : 64 * (step >> 1) + 8 * j;
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int col = col0 + e;
            float t = 0.0f;
            if (grow < p.M && col < p.r)
              t = __fmul_rn(p.lora[static_cast<size_t>(grow) * p.r + col], gprod);
            const float hi = __bfloat162float(__float2bfloat16_rn(t));
            v[e] = part == 0 ? hi : __fsub_rn(t, hi);
          }
          *reinterpret_cast<uint4*>(arow + ((j ^ (row & 7)) << 4)) =
              make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                         pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(lr_full);
    }
    if (mbar_wait(acc_full, 0, p.wait, kErrTimeoutAcc)) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < BN / 16; ++c) {
        uint32_t acc[16];
        tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(32 * quad) << 16) + c * 16, acc);
        tmem_ld_wait();
        const int col = n0 + c * 16;
        if (grow < p.M && col < p.N) {
          float o[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float b = p.bias ? __uint_as_float(static_cast<uint32_t>(p.bias[col + e]) << 16) : 0.0f;
            o[e] = __fadd_rn(__fmul_rn(__uint_as_float(acc[e]), alpha), b);
          }
          uint4* dst = reinterpret_cast<uint4*>(p.y + static_cast<size_t>(grow) * p.ldy + col);
          dst[0] = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                              pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
          dst[1] = make_uint4(pack_bf16x2(o[8], o[9]), pack_bf16x2(o[10], o[11]),
                              pack_bf16x2(o[12], o[13]), pack_bf16x2(o[14], o[15]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

template <int BN>
svdq_status launch_bn(const LaunchCtx& ctx, const CUtensorMap& ta, const CUtensorMap& tb,
                      const CUtensorMap& tl, const GemmParams& p) {
  using L = Layout<BN>;
  const size_t smem = 1024 + kStages * static_cast<size_t>(L::kStage) + 8 * (2 * kStages + 2) + 16;
  static bool attr_done[64] = {};
  if (!attr_done[ctx.device & 63]) {
    cudaFuncSetAttribute(w4a4_gemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
    attr_done[ctx.device & 63] = true;
  }
  dim3 grid((p.N + BN - 1) / BN, (p.M + kBM - 1) / kBM);
  w4a4_gemm_kernel<BN><<<grid, kThreads, smem, ctx.stream>>>(ta, tb, tl, p);
  return check_launch("w4a4_gemm_kernel");
}

}  // namespace

svdq_status launch_w4a4_gemm(const LaunchCtx& ctx, const uint8_t* q_act, const uint8_t* sf_act,
                             const float* act_gscale, const float* lora_act, const uint8_t* q_w,
                             const uint8_t* sf_w, const float* w_gscale, const void* L2t, int r,
                             const void* bias, int64_t M, int64_t N, int64_t K, void* y,
                             int64_t ldy) {
  const int bn = (N % 256 == 0) ? 256 : 128;
  CUtensorMap ta{}, tb{}, tl{};
  if (!make_tmap_2d(&ta, q_act, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, K / 2, K / 2, kBM, kBKBytes,
                    128))
    return SVDQ_ERR_CUDA;
  if (!make_tmap_2d(&tb, q_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / 2, K / 2, bn, kBKBytes, 128))
    return SVDQ_ERR_CUDA;
  if (r > 0) {
    if (!make_tmap_2d(&tl, L2t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, r, static_cast<uint64_t>(r) * 2,
                      bn, 64, 128))
      return SVDQ_ERR_CUDA;
  } else {
    tl = ta;
  }
  GemmParams p{};
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.r = r;
  p.bn = bn;
  p.sf_a = sf_act;
  p.sf_w = sf_w;
  p.gs_a = act_gscale;
  p.gs_w = w_gscale;
  p.lora = lora_act;
  p.bias = static_cast<const uint16_t*>(bias);
  p.y = static_cast<uint16_t*>(y);
  p.ldy = ldy;
  p.fault = ctx.fault_flags;
  p.wait = WaitCfg{ctx.timeout_ns, ctx.err_word};
  return bn == 256 ? launch_bn<256>(ctx, ta, tb, tl, p) : launch_bn<128>(ctx, ta, tb, tl, p);
}

}  // namespace svdq
