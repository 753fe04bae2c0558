// gemm.cu — svdq_w4a4_linear: the NVFP4 W4A4 GEMM with the low-rank
// up-projection fused in ("the low-rank up-projection is fused with the
// 4-bit compute kernel", blog.margrop.com "技术细节 §1", SVDQuant step 4).
//
//   y = bf16( α·acc + bias ),  α = 1/(gs_a·gs_w)
//   acc = Σ_k e2m1_a·sfa · e2m1_w·sfw      (kind::mxf4nvf4 block-scaled MMAs)
//       + (hi + lo)·L2                      (kind::f16 MMAs, same accumulator)
//   hi = bf16(xl·gs_a·gs_w), lo = bf16(xl·gs_a·gs_w − hi)
// The low-rank term can dominate y (it carries the outlier channels), so
// its activation operand keeps ~16 significant bits through the hi/lo
// split; L2 itself is bf16 by construction.
//
// Persistent kernel: one CTA per SM walks 128 x BN output tiles (BN = 256,
// or 128 when N is not a multiple of 256); fp32 accumulator in TMEM.
//   warp 0     producer.  For each tile: the FP4 steps (TMA of 128-byte rows
//              of packed A and B = 256 K-elements, 128-byte swizzle; bulk
//              copies of the matching scale blocks — the 128x4 block layout
//              is already the byte order the scale copy to TMEM wants),
//              then the low-rank steps (TMA of a 64-wide slice of L2ᵀ).
//              All go through one kStages-deep shared-memory ring.
//   warp 1     TMEM owner and MMA issuer (one thread).  Per FP4 step:
//              tcgen05.cp of the scale blocks into TMEM (4 columns per 128
//              rows per 64 K), four block-scaled MMAs (K = 64 each).  Per
//              low-rank step: kind::f16 MMAs into the same accumulator.
//              tcgen05.commit frees ring slots and, after a tile's last
//              step, hands the accumulator to the epilogue.
//   warps 2-9  epilogue, two warps per 32-lane TMEM quadrant (one per half
//              of BN).  During a tile's mainloop they write the tile's
//              low-rank A operand (hi/lo bf16 of the fp32 down-projection,
//              swizzled by hand) into the ring slots of its low-rank steps
//              and stage the bias slice in shared memory; after the
//              accumulator is full they drain TMEM -> registers (α·acc +
//              bias -> bf16), release the accumulator to the MMA warp and
//              store y while the next tile's mainloop runs.
#include "internal.h"
#include "ptx.cuh"

namespace svdq {
namespace {

constexpr int kBM = 128;
constexpr int kBKBytes = 128;  // 256 FP4 elements per FP4 step and row
constexpr int kStages = 4;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr uint32_t kATileBytes = kBM * kBKBytes;  // 16 KB

struct GemmParams {
  int M, N, K, r;
  int tiles_n, tiles;     // output tiles along N, total
  const uint8_t* sf_a;
  const uint8_t* sf_w;
  const float* gs_a;
  const float* gs_w;
  const float* lora;      // [M, r]
  const uint16_t* bias;   // [N] or null
  uint16_t* y;
  int64_t ldy;
  int fault;              // test hook: 1 = the first ring slot never fills
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
  static constexpr uint32_t kRing = kStages * kStage;
  static constexpr uint32_t kBias = kEpiWarps * (BN / 2) * 2;  // per-warp bias slices
  static constexpr uint32_t kTmemCols = BN == 256 ? 512 : 256;
  static constexpr uint32_t kSfaCol = BN;                // 16 columns
  static constexpr uint32_t kSfbCol = BN + 16;           // (BN/128)*16 columns
  static constexpr int kColsPerWarp = BN / 2;            // epilogue columns per warp
  static_assert(kStage % 1024 == 0, "stage must keep 1 KB alignment");
  static_assert(BN + 16 + (BN / 128) * 16 <= kTmemCols, "TMEM budget");
};

// Where tile `t` sits in the output.
__device__ __forceinline__ void tile_coords(int t, int tiles_n, int bn, int& m0, int& n0) {
  m0 = (t / tiles_n) * kBM;
  n0 = (t % tiles_n) * bn;
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                     const __grid_constant__ CUtensorMap tmap_b,
                     const __grid_constant__ CUtensorMap tmap_l2, const GemmParams p) {
  using L = Layout<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint16_t* bias_s = reinterpret_cast<uint16_t*>(base + L::kRing);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + L::kRing + L::kBias);
  uint64_t* empty = full + kStages;
  uint64_t* lrf = empty + kStages;       // low-rank A written, per ring slot
  // Slot free for a low-rank A write.  The epilogue cannot wait on empty[s]
  // for that: it looks several ring steps ahead, and a parity wait cannot
  // tell phase p from p + 2.  lrfree[s] completes one phase per low-rank use
  // of slot s (committed by the MMA when the slot's previous step is done),
  // so it can never run more than one phase ahead of the epilogue.
  uint64_t* lrfree = lrf + kStages;
  uint64_t* acc_full = lrfree + kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
  auto stage_a = [&](int s) { return base + s * L::kStage; };
  auto stage_b = [&](int s) { return base + s * L::kStage + kATileBytes; };
  auto stage_sfa = [&](int s) { return base + s * L::kStage + kATileBytes + L::kB; };
  auto stage_sfb = [&](int s) { return base + s * L::kStage + kATileBytes + L::kB + L::kSfa; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool lr_packed = p.r > 0 && p.r <= 32;  // hi and lo share one A tile
  const int nlr = p.r == 0 ? 0 : (lr_packed ? 1 : 2 * (p.r / 64));  // low-rank steps per tile
  const int kblocks = p.K / 64;              // 64-element K blocks (one MMA each)
  const int nk = (kblocks + 3) / 4;          // FP4 steps per tile (last may be short)
  const int nsteps = nk + nlr;               // ring steps per tile
  const int nb_total = (p.N + 127) / 128;    // 128-row blocks of the weight scales

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&lrf[s], kEpiWarps / 2);
      mbar_init(&lrfree[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kEpiWarps);
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
      int it = 0;          // ring step counter (continues across tiles)
      int issued_to = 0;   // ring steps whose loads were issued
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x) {
        int m0, n0;
        tile_coords(t, p.tiles_n, BN, m0, n0);
        const int nbl = min(BN / 128, nb_total - n0 / 128);  // weight scale row blocks
        for (int st = 0; st < nsteps; ++st, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, p.wait, kErrTimeoutEmpty)) {
            ok = false;
            break;
          }
          if (st < nk) {
            if (p.fault == 1 && it == 0) continue;  // test hook: this slot never fills
            const int kb = st;                      // 256-element K step
            const int nkb = min(4, kblocks - 4 * kb);
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
          } else {
            // L2ᵀ[n0 .. n0+BN) x r[64c .. 64c+64) as bf16, zero-filled past r
            const int j = st - nk;
            const int c = lr_packed ? 0 : j / 2;
            mbar_arrive_expect_tx(&full[s], L::kB);
            tma_load_2d(stage_b(s), &tmap_l2, &full[s], 64 * c, n0);
          }
          issued_to = it + 1;
        }
      }
      // never leave the CTA with a copy still landing in its shared memory
      for (int i = max(0, issued_to - kStages); i < issued_to; ++i) {
        if (p.fault == 1 && i == 0) continue;
        mbar_wait(&full[i % kStages], (i / kStages) & 1, p.wait, kErrTimeoutDrain);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA ----
    if (lane == 0) {
      const uint32_t id_f16 = idesc_f16(128, BN, true);
      const uint32_t id_fp4 = idesc_nvfp4(128, BN);
      int it = 0;
      uint32_t lr_par = 0;                   // parity of each slot's next low-rank phase
      int local = 0;                         // tiles done by this CTA
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x, ++local) {
        // the epilogue must have drained the previous tile's accumulator
        if (local > 0 && !mbar_wait(acc_empty, (local - 1) & 1, p.wait, kErrTimeoutAcc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int st = 0; st < nsteps; ++st, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!mbar_wait(&full[s], ph, p.wait, kErrTimeoutFull)) {
            ok = false;
            break;
          }
          const uint32_t a0 = smem_u32(stage_a(s));
          const uint32_t b0 = smem_u32(stage_b(s));
          if (st < nk) {
            tc_fence_after();
            const uint32_t sa = smem_u32(stage_sfa(s));
            const uint32_t sb = smem_u32(stage_sfb(s));
            const int nkb = min(4, kblocks - 4 * st);
            for (int kk = 0; kk < nkb; ++kk) {
              tmem_cp_32x128b_warpx4(tmem + L::kSfaCol + 4 * kk,
                                     make_sdesc(sa + kk * 512, 128, 128, kSwzNone));
#pragma unroll
              for (int nb = 0; nb < BN / 128; ++nb)
                tmem_cp_32x128b_warpx4(tmem + L::kSfbCol + (BN / 128) * 4 * kk + 4 * nb,
                                       make_sdesc(sb + (nb * 4 + kk) * 512, 128, 128, kSwzNone));
            }
            for (int kk = 0; kk < nkb; ++kk) {
              const uint64_t ad = make_sdesc(a0 + kk * 32, 16, 1024, kSwz128);
              const uint64_t bd = make_sdesc(b0 + kk * 32, 16, 1024, kSwz128);
              umma_nvfp4(tmem, ad, bd, id_fp4, tmem + L::kSfaCol + 4 * kk,
                         tmem + L::kSfbCol + (BN / 128) * 4 * kk, (st > 0 || kk > 0) ? 1u : 0u);
            }
          } else {
            if (!mbar_wait(&lrf[s], (lr_par >> s) & 1u, p.wait, kErrTimeoutFull)) {
              ok = false;
              break;
            }
            lr_par ^= 1u << s;
            tc_fence_after();
            // packed: A k-steps [0, r/16) hold hi and [2, 2 + r/16) hold lo,
            // both against B k-steps [0, r/16); unpacked: 4 k-steps per slot
            const int ksteps = lr_packed ? p.r / 16 : 4;
            for (int kk = 0; kk < ksteps; ++kk) {
              const uint64_t bd = make_sdesc(b0 + kk * 32, 16, 1024, kSwz128);
              umma_f16(tmem, make_sdesc(a0 + kk * 32, 16, 1024, kSwz128), bd, id_f16, 1u);
              if (lr_packed)
                umma_f16(tmem, make_sdesc(a0 + (2 + kk) * 32, 16, 1024, kSwz128), bd, id_f16, 1u);
            }
          }
          umma_commit(&empty[s]);
          // the step kStages ahead reuses this slot; if it is a low-rank step,
          // tell the epilogue when this step's reads of the slot are done
          if ((it + kStages) % nsteps >= nk) umma_commit(&lrfree[s]);
        }
        if (ok) umma_commit(acc_full);
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue ----
    const int ew = warp - 2;                 // 0..7
    const int quad = warp & 3;               // TMEM lane quadrant this warp may access
    const int half = ew >> 2;                // which half of BN
    const int row = 32 * quad + lane;        // tile row == TMEM lane
    const float gprod = __fmul_rn(*p.gs_a, *p.gs_w);
    const float alpha = __fdiv_rn(1.0f, gprod);
    constexpr int kCols = L::kColsPerWarp;
    int it = 0;
    uint32_t free_par = 0;                   // parity of each slot's next lrfree phase
    int local = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x, ++local) {
      int m0, n0;
      tile_coords(t, p.tiles_n, BN, m0, n0);
      const int grow = m0 + row;
      // (1) this warp's bias slice into its own shared-memory buffer (only
      // this warp reads it, after the __syncwarp below, and it rewrites it
      // only after its previous drain finished reading it)
      uint16_t* bsl = bias_s + ew * kCols;
      for (int c = lane; c < kCols; c += 32) {
        const int col = n0 + half * kCols + c;
        bsl[c] = (p.bias && col < p.N) ? p.bias[col] : static_cast<uint16_t>(0);
      }
      __syncwarp();
      // (2) the low-rank A operand of this tile, into the ring slots of its
      // low-rank steps (they follow the tile's FP4 steps); one warp per
      // quadrant writes its 32 rows
      it += nk;
      for (int j = 0; j < nlr; ++j, ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        (void)ph;
        if (half != 0) continue;
        if (it >= kStages) {  // the slot had a previous user: wait until it is done
          if (!mbar_wait(&lrfree[s], (free_par >> s) & 1u, p.wait, kErrTimeoutEmpty)) {
            ok = false;
            break;
          }
          free_par ^= 1u << s;
        }
        uint8_t* arow = stage_a(s) + row * 128;
#pragma unroll
        for (int q = 0; q < 8; ++q) {  // 8 bf16 = one 16-byte chunk
          // packed: chunks 0-3 = hi of columns 0..31, chunks 4-7 = lo of them;
          // unpacked: slice j/2, part j%2 (0 = hi, 1 = lo)
          const int part = lr_packed ? (q >> 2) : (j & 1);
          const int col0 = lr_packed ? 8 * (q & 3) : 64 * (j >> 1) + 8 * q;
          float v[8];
          if (grow < p.M && col0 < p.r) {
            const float4* src =
                reinterpret_cast<const float4*>(p.lora + static_cast<size_t>(grow) * p.r + col0);
            const float4 u0 = src[0], u1 = src[1];
            const float w8[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float tv = __fmul_rn(w8[e], gprod);
              const float hi = __bfloat162float(__float2bfloat16_rn(tv));
              v[e] = part == 0 ? hi : __fsub_rn(tv, hi);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = 0.0f;
          }
          *reinterpret_cast<uint4*>(arow + ((q ^ (row & 7)) << 4)) =
              make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                         pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&lrf[s]);
      }
      if (!ok) break;
      // (3) drain the accumulator: α·acc + bias -> packed bf16 in registers
      if (!mbar_wait(acc_full, local & 1, p.wait, kErrTimeoutAcc)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t packed[kCols / 2];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * quad) << 16) + half * kCols;
#pragma unroll
      for (int c = 0; c < kCols / 16; c += 2) {
        uint32_t a0[16], a1[16];
        tmem_ld_32x32b_x16(taddr + c * 16, a0);
        tmem_ld_32x32b_x16(taddr + (c + 1) * 16, a1);
        tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const uint32_t* a = u ? a1 : a0;
          const uint4* b4 = reinterpret_cast<const uint4*>(bsl + (c + u) * 16);
          const uint4 bb0 = b4[0], bb1 = b4[1];
          const uint32_t bw[8] = {bb0.x, bb0.y, bb0.z, bb0.w, bb1.x, bb1.y, bb1.z, bb1.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float lo = __fadd_rn(__fmul_rn(__uint_as_float(a[2 * e]), alpha),
                                       __uint_as_float(bw[e] << 16));
            const float hi = __fadd_rn(__fmul_rn(__uint_as_float(a[2 * e + 1]), alpha),
                                       __uint_as_float(bw[e] & 0xFFFF0000u));
            packed[(c + u) * 8 + e] = pack_bf16x2(lo, hi);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);   // the MMA may start the next tile
      // (4) store y (overlaps the next tile's mainloop)
      const int colb = n0 + half * kCols;
      if (grow < p.M) {
        uint4* dst = reinterpret_cast<uint4*>(p.y + static_cast<size_t>(grow) * p.ldy + colb);
#pragma unroll
        for (int q = 0; q < kCols / 8; ++q)
          if (colb + 8 * q < p.N)
            dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
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
                      const CUtensorMap& tl, GemmParams p) {
  using L = Layout<BN>;
  const size_t smem = 1024 + static_cast<size_t>(L::kRing) + L::kBias + 8 * (4 * kStages + 2) + 16;
  static bool attr_done[64] = {};
  if (!attr_done[ctx.device & 63]) {
    cudaFuncSetAttribute(w4a4_gemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
    attr_done[ctx.device & 63] = true;
  }
  p.tiles_n = (p.N + BN - 1) / BN;
  p.tiles = p.tiles_n * ((p.M + kBM - 1) / kBM);
  const int grid = std::min(p.tiles, ctx.num_sms);
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
    if (!make_tmap_2d(&tl, L2t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, r,
                      static_cast<uint64_t>(r) * 2, bn, 64, 128))
      return SVDQ_ERR_CUDA;
  } else {
    tl = ta;
  }
  GemmParams p{};
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.r = r;
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
