// gemm.cu — svdq_w4a4_linear: the NVFP4 W4A4 GEMM with the low-rank
// up-projection computed in the same kernel, into the same accumulator
// (blog.margrop.com "技术细节 §1", SVDQuant step 4: the pages pair the
// branch's up-projection with the 4-bit GEMM so it costs no extra pass).
//
//   y = bf16( α·acc + bias ),  α = 1/(gs_a·gs_w)
//   acc = Σ_k e2m1_a·sfa · e2m1_w·sfw      (kind::mxf4nvf4 block-scaled MMAs)
//       + (hi + lo)·L2                      (kind::f16 MMAs, same accumulator)
//   hi = bf16(xl·gs_a·gs_w), lo = bf16(xl·gs_a·gs_w − hi)
// The low-rank term can dominate y (it carries the outlier channels), so
// its activation operand keeps ~16 significant bits through the hi/lo
// split; L2 itself is bf16 by construction.
//
// Persistent kernel: one CTA per SM walks 128 x BN output tiles (BN = 192
// when N is a multiple of 192, else 128).  Tensor memory holds two fp32
// accumulators (the epilogue drains one while the MMAs fill the other) and
// a ring of scale-factor regions (the stagers fill regions ahead of the MMAs
// that read them): 3 regions of 40 columns at BN = 192, 8 of 32 at BN = 128.
//   warps 0-1   producers (slot s of the kStages-deep ring belongs to warp
//               s % 2): per FP4 step (256 K) bulk copies of the step's
//               128x4 scale blocks (on their own barrier, so the stagers can
//               start while the operands land), then TMA of packed A (128
//               rows x 128 B) and B (BN rows x 128 B) with 128-byte swizzle; per
//               low-rank step (32 of the r columns) TMA of the L2ᵀ slice and
//               of the tile's fp32 xl slice (into the A slot).  A thread that
//               issues copies spends a few hundred cycles per barrier round,
//               so two threads share the work.
//   warp 2      TMEM owner and MMA issuer (one thread): four block-scaled
//               MMAs (K = 64 each) per FP4 step, then the low-rank kind::f16
//               MMAs, into the tile's accumulator; tcgen05.commit frees ring
//               slots and scale regions and, at the end of a tile, hands the
//               accumulator to the epilogue.  It waits on one barrier per
//               step and does nothing else: the tensor pipe holds about one
//               MMA ahead, so latency in the issuing thread idles it.
//   warps 3-6   stagers, one per 32-lane TMEM quadrant.  Per FP4 step they
//               read the step's E4M3 scales from the ring slot and write them
//               into a scale region with tcgen05.st, every quadrant holding
//               the same copy (lane l, column j: the 4 scales of row 32j + l
//               per 64-K block, the order the block-scaled MMA reads).  Stores from registers run
//               beside the MMAs; a shared-to-TMEM copy issued by the MMA
//               thread would queue behind them.  Per low-rank step they turn
//               the slot's xl slice in place into the low-rank A operand: 32
//               columns of hi and 32 of lo (bf16 of xl·gs_a·gs_w and of its
//               remainder), swizzled by hand.
//   warps 7-10  epilogue, one per quadrant: per 64-column box, TMEM ->
//               registers (α·acc + bias [-> GELU] -> bf16) -> a 32 x 64
//               staging box in shared memory -> TMA store (full-line writes,
//               clipped at the M and N edges) into the tile's output (one,
//               or one of up to three parts: Q, K, V of a fused
//               projection); then release the accumulator.
// Every CTA initialises its barriers, allocates tensor memory and prefetches
// its descriptors before griddepcontrol.wait, so with programmatic dependent
// launch that set-up overlaps the previous kernel's tail.  A step needs 46
// KB of operands per SM from L2 at BN = 192, more than TMA delivers in the
// 384 cycles of its four MMAs when every SM streams: the operand feed, not
// the tensor pipe, sets the step time.
#include "gemm_common.cuh"

namespace svdq {
namespace {

constexpr int kBM = 128;
constexpr int kBKBytes = kGemmBKBytes;
constexpr int kStages = 4;                 // ring slots
constexpr int kProducers = 2;              // producer warps; slot s belongs to producer s % 2
constexpr int kMmaWarp = kProducers;
constexpr int kStagerWarps = 4;
constexpr int kEpiWarps = 4;
// 11 warps: at most 3 per SM sub-partition, so up to 168 registers a thread
constexpr int kThreads = 32 * (kProducers + 1 + kStagerWarps + kEpiWarps);
constexpr uint32_t kATileBytes = kBM * kBKBytes;  // 16 KB
constexpr int kMaxRegions = 8;

template <int BN>
struct Layout {
  static constexpr uint32_t kB = BN * kBKBytes;          // B tile bytes
  static constexpr uint32_t kSfa = 4 * 512;              // 4 K-blocks x 128 rows
  static constexpr uint32_t kSfb = (BN > 128 ? 2 : 1) * 4 * 512;  // one or two 128-row blocks
  static constexpr uint32_t kStage = kATileBytes + kB + kSfa + kSfb;
  static constexpr uint32_t kRing = kStages * kStage;
  static constexpr int kBoxes = BN / 64;                 // 64-column store boxes per tile
  static constexpr uint32_t kBoxBytes = 32 * 128;        // 32 rows x 64 bf16
  static constexpr uint32_t kBias = kEpiWarps * BN * 2;  // per-warp bias copies
  // A scale region holds one FP4 step's scales: SFA (4 columns per 64-K
  // block) at 4kk, SFB (BN/32 columns per block) at 16 + (BN/32)kk.  As
  // many regions as fit after the two accumulators: a region is rewritten
  // only after the MMAs that read it completed, and that completion reaches
  // the stagers about two steps after the MMAs were issued.
  static constexpr uint32_t kSfbCols = BN / 32;
  static constexpr uint32_t kSfRegionCols = 16 + 4 * kSfbCols;
  static constexpr uint32_t kSfCol = 2 * BN;             // first scale-region column
  static constexpr int kRegions = (512 - 2 * BN) / kSfRegionCols;
  static_assert(kStage % 1024 == 0, "stage must keep 1 KB alignment");
  static_assert(kRegions >= 3 && kRegions <= kMaxRegions, "TMEM budget");
  static_assert(BN % 64 == 0 && BN <= 256, "tile width");
};

// Where tile `t` sits in the output.
__device__ __forceinline__ void tile_coords(int t, int tiles_n, int bn, int& m0, int& n0) {
  m0 = (t / tiles_n) * kBM;
  n0 = (t % tiles_n) * bn;
}

template <int BN, int ACT>
__global__ void __launch_bounds__(kThreads, 1)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                     const __grid_constant__ CUtensorMap tmap_b,
                     const __grid_constant__ CUtensorMap tmap_l2,
                     const __grid_constant__ CUtensorMap tmap_y,
                     const __grid_constant__ CUtensorMap tmap_lr,
                     const __grid_constant__ CUtensorMap tmap_y1,
                     const __grid_constant__ CUtensorMap tmap_y2, const GemmParams p) {
  using L = Layout<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* out_s = base + L::kRing;                                     // [kEpiWarps][box]
  uint16_t* bias_s = reinterpret_cast<uint16_t*>(out_s + kEpiWarps * L::kBoxBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(bias_s) + L::kBias);
  uint64_t* full_sf = full + kStages;    // the slot's scale blocks landed (FP4 steps)
  uint64_t* empty = full_sf + kStages;
  uint64_t* lrf = empty + kStages;       // low-rank A written, per ring slot
  uint64_t* sfready = lrf + kStages;     // [kRegions] scale region written (and the slot's operands landed)
  uint64_t* sffree = sfready + kMaxRegions;  // [kRegions] scale region read by its MMAs
  uint64_t* acc_full = sffree + kMaxRegions; // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  auto stage_a = [&](int s) { return base + s * L::kStage; };
  auto stage_b = [&](int s) { return base + s * L::kStage + kATileBytes; };
  auto stage_sfa = [&](int s) { return base + s * L::kStage + kATileBytes + L::kB; };
  auto stage_sfb = [&](int s) { return base + s * L::kStage + kATileBytes + L::kB + L::kSfa; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // low-rank steps per tile: 32 columns of r each (r = 16: one, zero-padded)
  const int nlr = p.r == 0 ? 0 : (p.r <= 32 ? 1 : p.r / 32);
  const int kblocks = p.K / 64;              // 64-element K blocks (one MMA each)
  const int nk = (kblocks + 3) / 4;          // FP4 steps per tile (the last may be short)
  const int nsteps = nk + nlr;               // ring steps per tile

  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&full_sf[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&lrf[s], kStagerWarps);
    }
    for (int b = 0; b < L::kRegions; ++b) {
      mbar_init(&sfready[b], kStagerWarps);
      mbar_init(&sffree[b], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
    }
    fence_mbar_init();
  }
  if (warp == kMmaWarp && lane == 0) {
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b);
    if (p.r > 0) tma_prefetch_desc(&tmap_l2);
    if (p.r > 0) tma_prefetch_desc(&tmap_lr);
    tma_prefetch_desc(&tmap_y);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // global memory only after the previous kernel on the stream is done

  if (warp < kProducers) {
    // ------------------------------------------------------ producers ----
    if (lane == 0) {
      int it = 0;              // ring step counter (continues across tiles)
      uint32_t used = 0;       // slots this thread loaded
      uint32_t last_par = 0;   // per slot: parity of the last phase armed
      uint32_t sf_used = 0;    // slots this thread loaded scales into
      uint32_t sf_par = 0;     // per slot: parity of the next full_sf phase
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x) {
        int m0, n0;
        tile_coords(t, p.tiles_n, BN, m0, n0);
        for (int st = 0; st < nsteps; ++st, ++it) {
          const int s = it % kStages;
          if (s % kProducers != warp) continue;
          const uint32_t ph = (it / kStages) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, p.wait, kErrTimeoutEmpty)) {
            ok = false;
            break;
          }
          if (st < nk) {
            if (p.fault == 1 && it == 0) continue;  // test hook: this slot never fills
            const int nkb = min(4, kblocks - 4 * st);
            const uint32_t sfbytes = static_cast<uint32_t>(nkb) * 512;
            const size_t koff = static_cast<size_t>(4 * st) * 512;
            const uint8_t* wsf = p.sf_w + static_cast<size_t>(n0 / 128) * kblocks * 512 + koff;
            mbar_arrive_expect_tx(&full_sf[s], sfbytes * (BN > 128 ? 3 : 2));
            bulk_load(stage_sfa(s), p.sf_a + static_cast<size_t>(m0 / 128) * kblocks * 512 + koff,
                      sfbytes, &full_sf[s]);
            bulk_load(stage_sfb(s), wsf, sfbytes, &full_sf[s]);
            if (BN > 128) bulk_load(stage_sfb(s) + 2048, wsf + static_cast<size_t>(kblocks) * 512, sfbytes, &full_sf[s]);
            sf_used |= 1u << s;
            sf_par ^= 1u << s;
            mbar_arrive_expect_tx(&full[s], kATileBytes + L::kB);
            tma_load_2d(stage_a(s), &tmap_a, &full[s], st * kBKBytes, m0);
            tma_load_2d(stage_b(s), &tmap_b, &full[s], st * kBKBytes, n0);
          } else {
            // L2ᵀ[n0 .. n0+BN) x r[32j .. 32j+64) as bf16 (only the first 32
            // columns are used) and xl[m0 .. m0+128) x r[32j .. 32j+32) as
            // fp32; both zero-filled past M, N and r
            const int j = st - nk;
            mbar_arrive_expect_tx(&full[s], L::kB + kATileBytes);
            tma_load_2d(stage_b(s), &tmap_l2, &full[s], 32 * j, n0);
            tma_load_2d(stage_a(s), &tmap_lr, &full[s], 32 * j, m0);
          }
          used |= 1u << s;
          last_par = (last_par & ~(1u << s)) | (ph << s);
        }
      }
      // never leave the CTA with a copy still landing in its shared memory:
      // an earlier phase of a slot completed before the slot was armed again
      for (int s = 0; s < kStages; ++s) {
        if (used & (1u << s)) mbar_wait(&full[s], (last_par >> s) & 1u, p.wait, kErrTimeoutDrain);
        if (sf_used & (1u << s))
          mbar_wait(&full_sf[s], ((sf_par >> s) & 1u) ^ 1u, p.wait, kErrTimeoutDrain);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA ----
    if (lane == 0) {
      const uint32_t id_f16 = idesc_f16(128, BN, true);
      const uint32_t id_fp4 = idesc_nvfp4(128, BN);
      // descriptors of slot 0, k-offset 0; a slot / k offset adds (bytes >> 4)
      // to the start-address field (shared addresses stay below 256 KB)
      const uint64_t da0 = make_sdesc(smem_u32(stage_a(0)), 16, 1024, kSwz128);
      const uint64_t db0 = make_sdesc(smem_u32(stage_b(0)), 16, 1024, kSwz128);
      // Everything below is kept incremental (no divisions, unrolled MMAs):
      // the tensor pipe holds about one MMA ahead of this thread, so scalar
      // latency between MMAs is idle tensor time.
      int s = 0;                             // ring slot of the next step
      uint64_t soff = 0;                     // its descriptor offset (bytes >> 4)
      int rg = 0;                            // scale region of the next FP4 step
      uint32_t sfr = tmem + L::kSfCol;       // its first column
      uint32_t sf_par = 0;                   // parity of each region's next sfready phase
      uint32_t lr_par = 0;                   // parity of each slot's next lrf phase
      const int nkb_last = kblocks - 4 * (nk - 1);  // 64-K blocks of the last FP4 step
      const int nk_full = nkb_last == 4 ? nk : nk - 1;  // FP4 steps of four MMAs
      const int lr_k = p.r < 32 ? 1 : 2;     // low-rank k-steps per slice (hi and lo each)
      static_assert((kStages & (kStages - 1)) == 0, "the ring index wraps by a mask");
      auto advance = [&]() {
        s = (s + 1) & (kStages - 1);
        soff = static_cast<uint64_t>(s) * (L::kStage >> 4);
      };
      // the stagers arrive only after the slot's operands have landed
      auto wait_scales = [&](bool ready) -> bool {
        if (!ready && !mbar_wait(&sfready[rg], (sf_par >> rg) & 1u, p.wait, kErrTimeoutFull)) return false;
        sf_par ^= 1u << rg;
        tc_fence_after();
        return true;
      };
      auto next_region = [&]() {
        rg = rg + 1 == L::kRegions ? 0 : rg + 1;
        sfr = tmem + L::kSfCol + static_cast<uint32_t>(rg) * L::kSfRegionCols;
      };
      int local = 0;                         // tiles done by this CTA
      bool ok = true;
      bool ready = false;                    // the next FP4 step's sfready phase is known complete
      for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x, ++local) {
        const int a = local & 1;
        const uint32_t acc = tmem + a * BN;
        // the epilogue must have drained this accumulator's previous tile
        if (local >= 2 &&
            !mbar_wait(&acc_empty[a], ((local >> 1) - 1) & 1, p.wait, kErrTimeoutAcc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // Full FP4 steps: straight-line code between the MMAs (a branch in
        // the MMA stream costs tensor time even when it is not taken).  The
        // next step's barrier is tested while the pipe is busy; a phase seen
        // complete stays complete, across tiles too.
        for (int st = 0; st < nk_full; ++st) {
          if (!wait_scales(ready)) {
            ok = false;
            break;
          }
          const uint64_t da = da0 + soff, db = db0 + soff;
          const int rg_next = rg + 1 == L::kRegions ? 0 : rg + 1;
          umma_nvfp4(acc, da, db, id_fp4, sfr, sfr + 16, st > 0 ? 1u : 0u);
          umma_nvfp4(acc, da + 2, db + 2, id_fp4, sfr + 4, sfr + 16 + L::kSfbCols, 1u);
          umma_nvfp4(acc, da + 4, db + 4, id_fp4, sfr + 8, sfr + 16 + 2 * L::kSfbCols, 1u);
          ready = mbar_test(&sfready[rg_next], (sf_par >> rg_next) & 1u);
          umma_nvfp4(acc, da + 6, db + 6, id_fp4, sfr + 12, sfr + 16 + 3 * L::kSfbCols, 1u);
          umma_commit(&empty[s]);
          umma_commit(&sffree[rg]);
          next_region();
          advance();
        }
        if (ok && nk_full < nk) {  // the short last FP4 step (K % 256 != 0)
          if (!wait_scales(ready)) {
            ok = false;
            break;
          }
          const uint64_t da = da0 + soff, db = db0 + soff;
          for (int kk = 0; kk < nkb_last; ++kk)
            umma_nvfp4(acc, da + 2 * kk, db + 2 * kk, id_fp4, sfr + 4 * kk, sfr + 16 + L::kSfbCols * kk,
                       (nk_full > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&empty[s]);
          umma_commit(&sffree[rg]);
          ready = false;
          next_region();
          advance();
        }
        if (!ok) break;
        for (int j = 0; ok && j < nlr; ++j) {
          if (!mbar_wait(&lrf[s], (lr_par >> s) & 1u, p.wait, kErrTimeoutFull)) {
            ok = false;
            break;
          }
          lr_par ^= 1u << s;
          tc_fence_after();
          // A k-steps {0, 1} hold hi and {2, 3} lo of the slice's 32
          // columns, both against B k-steps {0, 1} (r = 16: one of each)
          const uint64_t da = da0 + soff, db = db0 + soff;
          for (int kk = 0; kk < lr_k; ++kk) {
            umma_f16(acc, da + 2 * kk, db + 2 * kk, id_f16, 1u);
            umma_f16(acc, da + 2 * (2 + kk), db + 2 * kk, id_f16, 1u);
          }
          umma_commit(&empty[s]);
          advance();
        }
        if (ok) umma_commit(&acc_full[a]);
      }
    }
  } else if (warp < kMmaWarp + 1 + kStagerWarps) {  // stagers
    // ----------------------------------------------------------- stagers ----
    const int quad = warp & 3;               // TMEM lane quadrant this warp may access
    const int row = 32 * quad + lane;        // tile row of the low-rank A operand
    const uint32_t lane_off = static_cast<uint32_t>(32 * quad) << 16;
    const float gprod = __fmul_rn(*p.gs_a, *p.gs_w);
    int ss = 0;                              // ring slot of the next step
    uint32_t sph = 0;                        // its phase parity
    uint32_t sf_par = 0;                     // parity of each slot's next full_sf phase
    int f = 0;                               // FP4 steps done
    int rg = 0;                              // scale region of the next FP4 step
    uint32_t free_par = 0;                   // parity of each region's next sffree phase
    bool ok = true;
    // One FP4 step: the slot's scales into region rg (stage_scales).
    auto fp4_step = [&](bool hi64, int s, uint32_t ph) -> bool {
      // region rg's previous user is FP4 step f - kRegions
      if (f >= L::kRegions) {
        if (!mbar_wait(&sffree[rg], (free_par >> rg) & 1u, p.wait, kErrTimeoutEmpty)) return false;
        free_par ^= 1u << rg;
      }
      if (!mbar_wait(&full_sf[s], (sf_par >> s) & 1u, p.wait, kErrTimeoutFull)) return false;
      sf_par ^= 1u << s;
      tc_fence_after();
      stage_scales<BN>(stage_sfa(s), stage_sfb(s), lane, hi64, true,
                       tmem + lane_off + L::kSfCol + rg * L::kSfRegionCols);
      tmem_st_wait();
      tc_fence_before();
      // the MMA thread waits on sfready alone: make it imply the operands too
      if (!mbar_wait(&full[s], ph, p.wait, kErrTimeoutFull)) return false;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sfready[rg]);
      ++f;
      rg = rg + 1 == L::kRegions ? 0 : rg + 1;
      return true;
    };
    for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x) {
      int m0, n0;
      tile_coords(t, p.tiles_n, BN, m0, n0);
      const bool hi64 = (n0 & 127) != 0;
      for (int st = 0; ok && st < nsteps; ++st) {
        const int s = ss;
        const uint32_t ph = sph;
        if (++ss == kStages) {  // the ring position of the next step
          ss = 0;
          sph ^= 1u;
        }
        if (st < nk) {
          ok = fp4_step(hi64, s, ph);
        } else {
          // the tile's low-rank A operand, in place over the slot's xl slice
          if (!mbar_wait(&full[s], ph, p.wait, kErrTimeoutFull)) {
            ok = false;
            break;
          }
          lowrank_operand_row(stage_a(s) + row * 128, row, gprod);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&lrf[s]);
        }
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue ----
    const int ew = warp - (kMmaWarp + 1 + kStagerWarps);  // 0..3
    const int quad = warp & 3;               // TMEM lane quadrant this warp may access
    const float alpha = __fdiv_rn(1.0f, __fmul_rn(*p.gs_a, *p.gs_w));
    uint16_t* bsl = bias_s + ew * BN;
    uint8_t* box = out_s + ew * L::kBoxBytes;
    uint8_t* brow = box + lane * 128;
    constexpr bool gelu = ACT == SVDQ_ACT_GELU_TANH;
    int local = 0;                           // tiles drained
    for (int t = blockIdx.x; t < p.tiles; t += gridDim.x, ++local) {
      int m0, n0;
      tile_coords(t, p.tiles_n, BN, m0, n0);
      const int a = local & 1;
      int ycol;
      const CUtensorMap* ymap = output_map(p, n0, &tmap_y, &tmap_y1, &tmap_y2, ycol);
      // the tile's bias columns into this warp's shared-memory copy
      for (int c = lane; c < BN; c += 32) {
        const int col = n0 + c;
        bsl[c] = (p.bias && col < p.N) ? p.bias[col] : static_cast<uint16_t>(0);
      }
      __syncwarp();
      if (!mbar_wait(&acc_full[a], (local >> 1) & 1, p.wait, kErrTimeoutAcc)) break;
      tc_fence_after();
      const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * quad) << 16) + a * BN;
#pragma unroll 1
      for (int j = 0; j < L::kBoxes; ++j) {
        // α·acc + bias -> bf16 for columns [64j, 64j + 64) of this quadrant's rows
        uint32_t packed[32];
        epilogue_box<gelu>(taddr + 64 * j, bsl + 64 * j, alpha, packed);
        if (j == L::kBoxes - 1) {  // the accumulator is drained: the MMAs may refill it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[a]);
        }
        // 32 x 64 staging box, 128-byte swizzle
        if (lane == 0) bulk_wait_group_read<0>();  // the previous store has read the box
        __syncwarp();
        write_box(brow, lane, packed);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(ymap, box, ycol + 64 * j, m0 + 32 * quad);
          bulk_commit_group();
        }
      }
    }
    if (lane == 0) bulk_wait_group<0>();  // all of this warp's stores are complete
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int BN, int ACT>
svdq_status launch_bn(const LaunchCtx& ctx, const CUtensorMap& ta, const CUtensorMap& tb,
                      const CUtensorMap& tl, const CUtensorMap& ty, const CUtensorMap& tr,
                      const CUtensorMap& ty1, const CUtensorMap& ty2, GemmParams p) {
  using L = Layout<BN>;
  const size_t smem = 1024 + static_cast<size_t>(L::kRing) + kEpiWarps * L::kBoxBytes + L::kBias +
                      8 * (4 * kStages + 2 * kMaxRegions + 4) + 16;
  if (svdq_status e = set_smem_attr(ctx, reinterpret_cast<const void*>(w4a4_gemm_kernel<BN, ACT>),
                                    static_cast<int>(smem)))
    return e;
  p.tiles_n = (p.N + BN - 1) / BN;
  p.tiles = p.tiles_n * ((p.M + kBM - 1) / kBM);
  const int grid = std::min(p.tiles, ctx.num_sms);
  return launch_kernel(ctx, "w4a4_gemm_kernel", w4a4_gemm_kernel<BN, ACT>, dim3(grid), dim3(kThreads), smem, ta,
                       tb, tl, ty, tr, ty1, ty2, p);
}

}  // namespace

svdq_status launch_w4a4_gemm(const LaunchCtx& ctx, const uint8_t* q_act, const uint8_t* sf_act,
                             const float* act_gscale, const float* lora_act, const uint8_t* q_w,
                             const uint8_t* sf_w, const float* w_gscale, const void* L2t, int r,
                             const void* bias, int64_t M, int64_t N, int64_t K, int parts,
                             void* const* y_parts, int64_t ldy, int activation) {
  // the tile width must divide every part (parts > 1: N/parts is a multiple of 128)
  const int64_t n_part = N / parts;
  const int bn = (n_part % 192 == 0) ? 192 : 128;
  // 256-row tiles on SM pairs (when enabled) where the shape has at least
  // two row blocks: 256 x 192 where 192 divides the part, else 256 x 128
  const int pair_bn = n_part % 192 == 0 ? 192 : 128;
  const bool pair = ctx.gemm_pairs && M > kBM && n_part % pair_bn == 0;
  CUtensorMap ta{}, tb{}, tl{}, ty{}, tr{}, ty1{}, ty2{};
  if (!make_tmap_2d(&ta, q_act, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, K / 2, K / 2, kBM, kBKBytes,
                    128))
    return SVDQ_ERR_CUDA;
  // B (and L2ᵀ) boxes: the tile's rows, or on SM pairs the half each CTA loads
  const uint32_t b_rows = static_cast<uint32_t>(pair ? pair_bn / 2 : bn);
  if (!make_tmap_2d(&tb, q_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / 2, K / 2, b_rows, kBKBytes, 128))
    return SVDQ_ERR_CUDA;
  if (r > 0) {
    if (!make_tmap_2d(&tl, L2t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, r,
                      static_cast<uint64_t>(r) * 2, b_rows, 64, 128))
      return SVDQ_ERR_CUDA;
  } else {
    tl = ta;
  }
  if (r > 0) {
    // xl [M, r] fp32 in 128-row x 32-column boxes (zero past M and r)
    if (!make_tmap_2d(&tr, lora_act, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, M, r,
                      static_cast<uint64_t>(r) * 4, kBM, 32, 0))
      return SVDQ_ERR_CUDA;
  } else {
    tr = ta;
  }
  CUtensorMap* ymaps[3] = {&ty, &ty1, &ty2};
  for (int i = 0; i < parts; ++i)
    if (!make_tmap_2d(ymaps[i], y_parts[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, n_part,
                      static_cast<uint64_t>(ldy) * 2, 32, 64, 128))
      return SVDQ_ERR_CUDA;
  for (int i = parts; i < 3; ++i) *ymaps[i] = ty;
  GemmParams p{};
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.r = r;
  p.sf_a = sf_act;
  p.sf_w = sf_w;
  p.gs_a = act_gscale;
  p.gs_w = w_gscale;
  p.bias = static_cast<const uint16_t*>(bias);
  p.n_part = parts > 1 ? static_cast<int>(n_part) : 0;
  p.fault = ctx.fault_flags;
  p.wait = WaitCfg{ctx.timeout_ns, ctx.err_word};
  if (pair) return launch_w4a4_gemm_pair(ctx, ta, tb, tl, ty, tr, ty1, ty2, p, pair_bn, activation);
  if (activation == SVDQ_ACT_GELU_TANH)
    return bn == 192 ? launch_bn<192, SVDQ_ACT_GELU_TANH>(ctx, ta, tb, tl, ty, tr, ty1, ty2, p)
                     : launch_bn<128, SVDQ_ACT_GELU_TANH>(ctx, ta, tb, tl, ty, tr, ty1, ty2, p);
  return bn == 192 ? launch_bn<192, SVDQ_ACT_NONE>(ctx, ta, tb, tl, ty, tr, ty1, ty2, p)
                   : launch_bn<128, SVDQ_ACT_NONE>(ctx, ta, tb, tl, ty, tr, ty1, ty2, p);
}

}  // namespace svdq
