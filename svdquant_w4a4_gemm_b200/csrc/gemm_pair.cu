// gemm_pair.cu — the W4A4 GEMM of svdq_w4a4_linear on SM pairs: 256 x 192
// output tiles, each computed by a cluster of two CTAs (two SMs) with
// tcgen05 cta_group::2 MMAs, for N (or N / parts) a multiple of 192.  The
// arithmetic is that of the one-SM kernel in gemm.cu (block-scaled NVFP4
// MMAs, then the low-rank up-projection in the same accumulator; the pages
// pair that up-projection with the 4-bit GEMM so the 16-bit branch costs no
// extra pass, blog.margrop.com "技术细节 §1", SVDQuant step 4):
//
//   y = bf16( α·acc + bias ),  α = 1/(gs_a·gs_w)
//   acc = Σ_k e2m1_a·sfa · e2m1_w·sfw  +  (hi + lo)·L2
//
// Why pairs: an MMA of the pair reads A from both SMs (128 rows each) and B
// from both (96 of the tile's 192 columns each), so per SM and FP4 step the
// ring moves 16 KB of A, 12 KB of B and 6 KB of scales (34 KB) for the same
// tensor work that costs the one-SM kernel 46 KB (A 16 KB, B 24 KB, scales
// 6 KB): more steps fit in shared memory (6 instead of 4) and the copies in
// flight cover more of the load latency.
//
// Roles, per CTA (rank 0 = the even CTA, which issues the MMAs):
//   warps 0-1   producers: this CTA's 128 rows of A, its 96 rows of B (L2ᵀ on
//               low-rank steps), the scales of its A rows and of all 192 B
//               rows (each SM's tensor memory holds the B scales of the whole
//               tile), with plain TMA and bulk copies into its own shared
//               memory, on its own barriers.
//   warp 2      TMEM: both CTAs allocate the pair's 512 columns together; in
//               rank 0, one thread issues the pair MMAs and commits them to the
//               barriers of both CTAs (slot free, scale region free,
//               accumulator full), one commit per CTA.
//   warps 3-6   stagers: scales into this SM's tensor memory and the low-rank
//               A operand in place, then an arrival on rank 0's barrier
//               (count 8: four warps of each CTA), so the MMA thread's one
//               wait covers both SMs' data.
//   warps 7-10  epilogue: this SM's 128 accumulator rows -> bf16 -> TMA
//               store; the accumulator is released with an arrival on rank
//               0's barrier (count 8).
// Tensor memory per SM: two 192-column fp32 accumulators, then three scale
// regions of 40 columns (SFA 4 x 4, SFB 4 x 6).  A CTA whose 128 rows lie
// past M (the last pair of an odd number of row blocks) loads zero-filled A
// and zero scales and stores nothing.  Every wait is bounded; both CTAs meet
// at a cluster barrier before the tensor memory is freed and before either
// exits, after the last commit has reached both.
#include <mutex>

#include "gemm_common.cuh"

namespace svdq {
namespace {

constexpr int kBM = 128;                   // rows per CTA (256 per pair tile)
constexpr int kBKBytes = kGemmBKBytes;

constexpr int kProducers = 2;              // slot s belongs to producer warp s % 2
constexpr int kMmaWarp = kProducers;
constexpr int kStagerWarps = 4;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 32 * (kProducers + 1 + kStagerWarps + kEpiWarps);
constexpr uint32_t kA = kBM * kBKBytes;            // 16 KB
constexpr uint32_t kSfa = 4 * 512;                 // this CTA's row block, 4 K-blocks
constexpr uint32_t kBoxBytes = 32 * 128;           // 32 rows x 64 bf16

// Sizes of a pair tile 256 x BN (BN = 128 or 192).
template <int BN>
struct PairLayout {
  static constexpr int kBHalf = BN / 2;                      // B (and L2ᵀ) rows each CTA loads
  static constexpr uint32_t kB = kBHalf * kBKBytes;
  static constexpr int kSfbBlocks = BN > 128 ? 2 : 1;        // 128-row scale blocks under BN rows
  static constexpr uint32_t kSfb = kSfbBlocks * 4 * 512;
  static constexpr uint32_t kStage = kA + kB + kSfa + kSfb;
  static constexpr int kBoxes = BN / 64;                     // 64-column store boxes per tile
  static constexpr uint32_t kBias = kEpiWarps * BN * 2;      // per-warp bias copies
  static constexpr uint32_t kSfbCols = BN / 32;
  static constexpr uint32_t kSfRegionCols = 16 + 4 * kSfbCols;
  static constexpr uint32_t kSfCol = 2 * BN;                 // first scale-region column
  static constexpr int kRegions = (512 - 2 * BN) / kSfRegionCols;
  static constexpr size_t kFixed = 1024 + kEpiWarps * kBoxBytes + kBias + 16;
  // ring depth: as many stages as shared memory holds (barriers: 4 per stage, 2 per region, 5)
  static constexpr int kStages = static_cast<int>((227 * 1024 - kFixed - 8 * (2 * kRegions + 5)) / (kStage + 32));
  static constexpr uint32_t kRing = kStages * kStage;
  static constexpr int kBarriers = 4 * kStages + 2 * kRegions + 5;
  static constexpr size_t kSmemBytes = kFixed + kRing + 8 * kBarriers;
  static_assert(kStage % 1024 == 0, "stage must keep 1 KB alignment");
  static_assert(kRegions >= 3 && kRegions <= 8, "TMEM budget");
  static_assert(kStages >= 4 && kStages <= 8, "ring depth");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

template <int BN, int ACT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    w4a4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a,
                          const __grid_constant__ CUtensorMap tmap_b,
                          const __grid_constant__ CUtensorMap tmap_l2,
                          const __grid_constant__ CUtensorMap tmap_y,
                          const __grid_constant__ CUtensorMap tmap_lr,
                          const __grid_constant__ CUtensorMap tmap_y1,
                          const __grid_constant__ CUtensorMap tmap_y2, const GemmParams p) {
  using L = PairLayout<BN>;
  constexpr int kBN = BN, kBHalf = L::kBHalf, kStages = L::kStages, kRegions = L::kRegions,
                kBoxes = L::kBoxes;
  constexpr uint32_t kB = L::kB, kStage = L::kStage, kRing = L::kRing, kBias = L::kBias,
                     kSfbCols = L::kSfbCols, kSfRegionCols = L::kSfRegionCols, kSfCol = L::kSfCol;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* out_s = base + kRing;                                          // [kEpiWarps][box]
  uint16_t* bias_s = reinterpret_cast<uint16_t*>(out_s + kEpiWarps * kBoxBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(bias_s) + kBias);
  uint64_t* full_sf = full + kStages;      // the slot's scale blocks landed (this CTA)
  uint64_t* empty = full_sf + kStages;     // the slot's MMAs completed (committed to both CTAs)
  uint64_t* lrf = empty + kStages;         // rank 0: low-rank A written in both CTAs
  uint64_t* sfready = lrf + kStages;       // rank 0: scale region written and operands landed, both CTAs
  uint64_t* sffree = sfready + kRegions;   // the region's MMAs completed (both CTAs)
  uint64_t* acc_full = sffree + kRegions;  // [2] the tile's MMAs completed (both CTAs)
  uint64_t* acc_empty = acc_full + 2;      // [2] rank 0: both epilogues drained the accumulator
  uint64_t* done = acc_empty + 2;          // the MMA thread's last commit (both CTAs)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  auto stage_a = [&](int s) { return base + s * kStage; };
  auto stage_b = [&](int s) { return base + s * kStage + kA; };
  auto stage_sfa = [&](int s) { return base + s * kStage + kA + kB; };
  auto stage_sfb = [&](int s) { return base + s * kStage + kA + kB + kSfa; };

  const uint32_t rank = cluster_ctarank();
  const int cluster = static_cast<int>(blockIdx.x >> 1), nclusters = static_cast<int>(gridDim.x >> 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nlr = p.r == 0 ? 0 : (p.r <= 32 ? 1 : p.r / 32);  // low-rank steps (32 of r each)
  const int kblocks = p.K / 64;
  const int nk = (kblocks + 3) / 4;        // FP4 steps per tile (the last may be short)
  const int nsteps = nk + nlr;

  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&full_sf[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&lrf[s], 2 * kStagerWarps);
    }
    for (int b = 0; b < kRegions; ++b) {
      mbar_init(&sfready[b], 2 * kStagerWarps);
      mbar_init(&sffree[b], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * kEpiWarps);
    }
    mbar_init(done, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b);
    if (p.r > 0) tma_prefetch_desc(&tmap_l2);
    if (p.r > 0) tma_prefetch_desc(&tmap_lr);
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  // both CTAs' barriers are initialized and the allocation is done before
  // anyone arrives on the other CTA's barriers
  tc_fence_before();
  cluster_sync_all();
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
      for (int t = cluster; ok && t < p.tiles; t += nclusters) {
        const int mp = t / p.tiles_n, n0 = (t % p.tiles_n) * kBN;
        const int m0 = mp * 2 * kBM + static_cast<int>(rank) * kBM;
        const bool a_valid = m0 < p.M;  // else: A reads zero fill and no scales exist
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
            mbar_arrive_expect_tx(&full_sf[s], sfbytes * static_cast<uint32_t>(L::kSfbBlocks + (a_valid ? 1 : 0)));
            if (a_valid)
              bulk_load(stage_sfa(s), p.sf_a + static_cast<size_t>(m0 / 128) * kblocks * 512 + koff,
                        sfbytes, &full_sf[s]);
            bulk_load(stage_sfb(s), wsf, sfbytes, &full_sf[s]);
            if (L::kSfbBlocks > 1)
              bulk_load(stage_sfb(s) + 2048, wsf + static_cast<size_t>(kblocks) * 512, sfbytes, &full_sf[s]);
            sf_used |= 1u << s;
            sf_par ^= 1u << s;
            mbar_arrive_expect_tx(&full[s], kA + kB);
            tma_load_2d(stage_a(s), &tmap_a, &full[s], st * kBKBytes, m0);
            tma_load_2d(stage_b(s), &tmap_b, &full[s], st * kBKBytes, n0 + static_cast<int>(rank) * kBHalf);
          } else {
            // this CTA's 96 rows of L2ᵀ x r[32j .. 32j+64) (the first 32 columns
            // are used) and its 128 rows of xl x r[32j .. 32j+32), zero-filled
            // past M, N and r
            const int j = st - nk;
            mbar_arrive_expect_tx(&full[s], kB + kA);
            tma_load_2d(stage_b(s), &tmap_l2, &full[s], 32 * j, n0 + static_cast<int>(rank) * kBHalf);
            tma_load_2d(stage_a(s), &tmap_lr, &full[s], 32 * j, m0);
          }
          used |= 1u << s;
          last_par = (last_par & ~(1u << s)) | (ph << s);
        }
      }
      // never leave the CTA with a copy still landing in its shared memory
      for (int s = 0; s < kStages; ++s) {
        if (used & (1u << s)) mbar_wait(&full[s], (last_par >> s) & 1u, p.wait, kErrTimeoutDrain);
        if (sf_used & (1u << s))
          mbar_wait(&full_sf[s], ((sf_par >> s) & 1u) ^ 1u, p.wait, kErrTimeoutDrain);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------- MMA (rank 0) ----
    if (rank == 0 && lane == 0) {
      const uint32_t id_f16 = idesc_f16(2 * kBM, kBN, true);
      const uint32_t id_fp4 = idesc_nvfp4(2 * kBM, kBN);
      // descriptors of slot 0, k-offset 0 (the same offsets address the other
      // CTA's half); a slot / k offset adds (bytes >> 4) to the address field
      const uint64_t da0 = make_sdesc(smem_u32(stage_a(0)), 16, 1024, kSwz128);
      const uint64_t db0 = make_sdesc(smem_u32(stage_b(0)), 16, 1024, kSwz128);
      int s = 0;                             // ring slot of the next step
      uint64_t soff = 0;                     // its descriptor offset (bytes >> 4)
      int rg = 0;                            // scale region of the next FP4 step
      uint32_t sfr = tmem + kSfCol;          // its first column
      uint32_t sf_par = 0;                   // parity of each region's next sfready phase
      uint32_t lr_par = 0;                   // parity of each slot's next lrf phase
      const int nkb_last = kblocks - 4 * (nk - 1);
      const int lr_k = p.r < 32 ? 1 : 2;     // low-rank k-steps per slice (hi and lo each)
      auto advance = [&]() {
        if (++s == kStages) {
          s = 0;
          soff = 0;
        } else {
          soff += kStage >> 4;
        }
      };
      int local = 0;
      bool ok = true;
      for (int t = cluster; ok && t < p.tiles; t += nclusters, ++local) {
        const int a = local & 1;
        const uint32_t acc = tmem + a * kBN;
        if (local >= 2 &&
            !mbar_wait(&acc_empty[a], ((local >> 1) - 1) & 1, p.wait, kErrTimeoutAcc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        bool ready = false;
        for (int st = 0; st < nk; ++st) {
          if (!ready &&
              !mbar_wait(&sfready[rg], (sf_par >> rg) & 1u, p.wait, kErrTimeoutFull)) {
            ok = false;
            break;
          }
          sf_par ^= 1u << rg;
          tc_fence_after();
          const uint64_t da = da0 + soff, db = db0 + soff;
          const int rg_next = rg + 1 == kRegions ? 0 : rg + 1;
          if (st + 1 < nk || nkb_last == 4) {
            umma_nvfp4_pair(acc, da, db, id_fp4, sfr, sfr + 16, st > 0 ? 1u : 0u);
            umma_nvfp4_pair(acc, da + 2, db + 2, id_fp4, sfr + 4, sfr + 16 + kSfbCols, 1u);
            umma_nvfp4_pair(acc, da + 4, db + 4, id_fp4, sfr + 8, sfr + 16 + 2 * kSfbCols, 1u);
            // look at the next step's barrier while the tensor pipe is busy
            ready = st + 1 < nk && mbar_test(&sfready[rg_next], (sf_par >> rg_next) & 1u);
            umma_nvfp4_pair(acc, da + 6, db + 6, id_fp4, sfr + 12, sfr + 16 + 3 * kSfbCols, 1u);
          } else {
            ready = false;
            for (int kk = 0; kk < nkb_last; ++kk)
              umma_nvfp4_pair(acc, da + 2 * kk, db + 2 * kk, id_fp4, sfr + 4 * kk,
                              sfr + 16 + kSfbCols * kk, (st > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit_pair(&empty[s]);
          umma_commit_pair(&sffree[rg]);
          rg = rg_next;
          sfr = rg == 0 ? tmem + kSfCol : sfr + kSfRegionCols;
          advance();
        }
        for (int j = 0; ok && j < nlr; ++j) {
          if (!mbar_wait(&lrf[s], (lr_par >> s) & 1u, p.wait, kErrTimeoutFull)) {
            ok = false;
            break;
          }
          lr_par ^= 1u << s;
          tc_fence_after();
          // A k-steps {0, 1} hold hi and {2, 3} lo of the slice's 32 columns,
          // both against B k-steps {0, 1} (r = 16: one of each)
          const uint64_t da = da0 + soff, db = db0 + soff;
          for (int kk = 0; kk < lr_k; ++kk) {
            umma_f16_pair(acc, da + 2 * kk, db + 2 * kk, id_f16, 1u);
            umma_f16_pair(acc, da + 2 * (2 + kk), db + 2 * kk, id_f16, 1u);
          }
          umma_commit_pair(&empty[s]);
          advance();
        }
        if (ok) umma_commit_pair(&acc_full[a]);
      }
      // arrives once everything issued above has completed
      umma_commit_pair(done);
    }
  } else if (warp < kMmaWarp + 1 + kStagerWarps) {
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
    for (int t = cluster; ok && t < p.tiles; t += nclusters) {
      const int mp = t / p.tiles_n, n0 = (t % p.tiles_n) * kBN;
      const bool a_valid = mp * 2 * kBM + static_cast<int>(rank) * kBM < p.M;
      const bool hi64 = (n0 & 127) != 0;
      for (int st = 0; ok && st < nsteps; ++st) {
        const int s = ss;
        const uint32_t ph = sph;
        if (++ss == kStages) {
          ss = 0;
          sph ^= 1u;
        }
        if (st < nk) {
          // region rg's previous user is FP4 step f - kRegions
          if (f >= kRegions) {
            if (!mbar_wait(&sffree[rg], (free_par >> rg) & 1u, p.wait, kErrTimeoutEmpty)) {
              ok = false;
              break;
            }
            free_par ^= 1u << rg;
          }
          if (!mbar_wait(&full_sf[s], (sf_par >> s) & 1u, p.wait, kErrTimeoutFull)) {
            ok = false;
            break;
          }
          sf_par ^= 1u << s;
          tc_fence_after();
          stage_scales<kBN>(stage_sfa(s), stage_sfb(s), lane, hi64, a_valid,
                            tmem + lane_off + kSfCol + rg * kSfRegionCols);
          tmem_st_wait();
          tc_fence_before();
          // the MMA thread waits on sfready alone: make it imply the operands too
          if (!mbar_wait(&full[s], ph, p.wait, kErrTimeoutFull)) {
            ok = false;
            break;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(&sfready[rg], 0);
          ++f;
          rg = rg + 1 == kRegions ? 0 : rg + 1;
        } else {
          if (!mbar_wait(&full[s], ph, p.wait, kErrTimeoutFull)) {
            ok = false;
            break;
          }
          lowrank_operand_row(stage_a(s) + row * 128, row, gprod);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(&lrf[s], 0);
        }
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue ----
    const int ew = warp - (kMmaWarp + 1 + kStagerWarps);  // 0..3
    const int quad = warp & 3;               // TMEM lane quadrant this warp may access
    const float alpha = __fdiv_rn(1.0f, __fmul_rn(*p.gs_a, *p.gs_w));
    uint16_t* bsl = bias_s + ew * kBN;
    uint8_t* box = out_s + ew * kBoxBytes;
    uint8_t* brow = box + lane * 128;
    constexpr bool gelu = ACT == SVDQ_ACT_GELU_TANH;
    int local = 0;
    for (int t = cluster; t < p.tiles; t += nclusters, ++local) {
      const int mp = t / p.tiles_n, n0 = (t % p.tiles_n) * kBN;
      const int m0 = mp * 2 * kBM + static_cast<int>(rank) * kBM;
      const bool store = m0 + 32 * quad < p.M;  // this warp's 32 rows hold output rows
      const int a = local & 1;
      int ycol;
      const CUtensorMap* ymap = output_map(p, n0, &tmap_y, &tmap_y1, &tmap_y2, ycol);
      for (int c = lane; c < kBN; c += 32) {
        const int col = n0 + c;
        bsl[c] = (p.bias && col < p.N) ? p.bias[col] : static_cast<uint16_t>(0);
      }
      __syncwarp();
      if (!mbar_wait(&acc_full[a], (local >> 1) & 1, p.wait, kErrTimeoutAcc)) break;
      tc_fence_after();
      const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * quad) << 16) + a * kBN;
#pragma unroll 1
      for (int j = 0; j < kBoxes; ++j) {
        uint32_t packed[32];
        epilogue_box<gelu>(taddr + 64 * j, bsl + 64 * j, alpha, packed);
        if (j == kBoxes - 1) {  // the accumulator is drained: the MMAs may refill it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(&acc_empty[a], 0);
        }
        if (!store) continue;
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
  // the MMA thread's last commit reaches both CTAs only after every MMA and
  // commit before it: wait for it so that no commit lands in a CTA that left
  if (warp == kMmaWarp && lane == 0) mbar_wait(done, 0, p.wait, kErrTimeoutDrain);
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// Clusters of two that fit on the device at once (once per context).
int pair_clusters(const LaunchCtx& ctx, const void* kernel, size_t smem) {
  static std::mutex mu;
  static unsigned long long ctx_of[64] = {};
  static int n_of[64] = {};
  std::lock_guard<std::mutex> lk(mu);
  const int d = ctx.device & 63;
  if (ctx_of[d] != ctx.ctx_id || n_of[d] <= 0) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * (ctx.num_sms / 2));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = ctx.num_sms / 2;
    }
    n_of[d] = n;
    ctx_of[d] = ctx.ctx_id;
  }
  return n_of[d];
}

template <int BN, int ACT>
svdq_status launch_act(const LaunchCtx& ctx, const CUtensorMap& ta, const CUtensorMap& tb,
                       const CUtensorMap& tl, const CUtensorMap& ty, const CUtensorMap& tr,
                       const CUtensorMap& ty1, const CUtensorMap& ty2, GemmParams p) {
  using L = PairLayout<BN>;
  const void* fn = reinterpret_cast<const void*>(w4a4_gemm_pair_kernel<BN, ACT>);
  if (svdq_status e = set_smem_attr(ctx, fn, static_cast<int>(L::kSmemBytes))) return e;
  p.tiles_n = p.N / BN;
  p.tiles = p.tiles_n * ((p.M + 2 * kBM - 1) / (2 * kBM));
  const int clusters = std::min(p.tiles, pair_clusters(ctx, fn, L::kSmemBytes));
  return launch_kernel(ctx, "w4a4_gemm_pair_kernel", w4a4_gemm_pair_kernel<BN, ACT>, dim3(2 * clusters),
                       dim3(kThreads), L::kSmemBytes, ta, tb, tl, ty, tr, ty1, ty2, p);
}

}  // namespace

svdq_status launch_w4a4_gemm_pair(const LaunchCtx& ctx, const CUtensorMap& ta, const CUtensorMap& tb,
                                  const CUtensorMap& tl, const CUtensorMap& ty, const CUtensorMap& tr,
                                  const CUtensorMap& ty1, const CUtensorMap& ty2, GemmParams p,
                                  int bn, int activation) {
  if (bn == 192)
    return activation == SVDQ_ACT_GELU_TANH
               ? launch_act<192, SVDQ_ACT_GELU_TANH>(ctx, ta, tb, tl, ty, tr, ty1, ty2, p)
               : launch_act<192, SVDQ_ACT_NONE>(ctx, ta, tb, tl, ty, tr, ty1, ty2, p);
  return activation == SVDQ_ACT_GELU_TANH
             ? launch_act<128, SVDQ_ACT_GELU_TANH>(ctx, ta, tb, tl, ty, tr, ty1, ty2, p)
             : launch_act<128, SVDQ_ACT_NONE>(ctx, ta, tb, tl, ty, tr, ty1, ty2, p);
}

}  // namespace svdq
