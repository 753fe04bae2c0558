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
//                of L1ᵀ into a shared-memory ring as deep as shared memory
//                allows, up to 8 sub-tiles (the loads come from HBM, and the
//                ring must cover its latency).  The first loads of the ring
//                go out as soon as the other warps have issued their own
//                set-up loads (s and gs; behind the x stream they would
//                wait microseconds), while those warps compute RN(1/s) once
//                for every column this CTA's range touches.
//   warp 1       TMEM owner; one thread issues the down-projection as
//                tcgen05 kind::f16 MMAs (M = 128, N = r, K = 16 each) from
//                the quantized tile's bf16(x̂) and the L1ᵀ slice into a TMEM
//                accumulator; a new accumulator (of two) per run of
//                sub-tiles in the same 128-row block ("segment").
//   warps 2-9    quantizers, two warps per sub-tile (64 rows each), so up
//                to ns/2 sub-tiles are worked on at once and a CTA's 10-11
//                sub-tiles split into ~21 half-tiles: the last round is half
//                as long.  Warp pair pq takes ring items pq, pq + ns/2, ...
//                in slots i mod ns: a pair owns two slots, and the previous
//                phase of every barrier it waits on is one it consumed itself
//                (a parity wait cannot tell a phase from the one two before
//                it, so a warp must never wait on a slot whose previous load
//                may still be outstanding).  The pair agrees on each wait's
//                verdict and meets before one of its warps releases the slot.
//                Lane l takes rows 64h + l and 64h + l + 32 and each row's
//                four 16-element groups: x̂ = x·inv_s (packed f32x2 products),
//                group max, E4M3 scale (RN(amax/6) by one Markstein correction
//                step, cvt.rn.satfinite.e4m3x2; RN(gs / scale) from a per-CTA
//                table of the 127 scale codes), E2M1 codes (cvt.rn.satfinite
//                .e2m1x2), the row's 32 code bytes and 4 scale bytes (one
//                word in the 128x4 block layout), and bf16(x̂) written back
//                over the tile for the MMA.
//   warps 10-13  epilogue: when a segment's accumulator is complete, TMEM ->
//                registers -> float4 atomics into xl (zeroed beforehand:
//                a row block's K range can span several CTAs), then release
//                the accumulator.
// HBM traffic is the algorithmic minimum: x once, codes + scales + xl once;
// L1ᵀ slices come from L2.  xl is cleared by a small kernel launched just
// before (clear_kernel, chained by programmatic dependent launch), and each
// quantizer warp writes its 32 rows of codes through a shared-memory staging
// area, so that a store covers whole 32-byte rows.
//
// Single-pass dynamic scale (gs_a = 2688 / max|x̂| computed in the same
// launch): every CTA first streams its sub-tiles once for the max (phase A;
// the quantizer warps take the sub-tiles as in phase B and release each
// slot straight away), folds its max into a global word, and meets the
// other CTAs at a grid barrier (cooperative launch, bounded wait); then
// phase B quantizes as above with the tensor-wide gs_a, reading x again,
// now from L2 (the CTA's phase-B loads go out while it waits at the
// barrier).  The ring runs through both phases as one sequence of 2n
// items, item i in slot i mod ns, taken by quantizer warp pair i mod ns/2.
#include <cstdio>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace svdq {
namespace {

constexpr int kBM = 128;
constexpr int kSubK = 64;
constexpr int kQuantWarps = 8;   // two per sub-tile, so up to 4 in flight
constexpr int kMaxStages = kQuantWarps;  // ring depth <= quantizer warps: two slots per warp pair
constexpr int kEpiWarps = 4;
constexpr int kThreads = 32 * (2 + kQuantWarps + kEpiWarps);
constexpr uint32_t kXTileBytes = kBM * kSubK * 2;

struct QuantParams {
  int M, K, r;
  int units;              // ceil(M/128) * (K/64) sub-tiles
  int stages;             // ring depth, 2 .. kMaxStages; also the number of working quantizer warps
  const float* smooth_s;  // [K] or null
  const float* gs_in;     // static tensor scale, or null for dynamic
  const float* amax_src;  // dynamic: amax bits (written by the amax pass)
  float* gs_copy;         // static: where to copy gs (block 0), or null
  uint8_t* q_out;
  uint8_t* sf_out;
  float* lora_out;
  uint32_t* sync;         // single-pass dynamic scale: [0] CTAs arrived, [1] max|x̂| bits, zero at launch
  int fault;              // test hook: bit 2 = CTA 0 never arrives at the grid barrier
  WaitCfg wait;
};

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float tensor_scale_from_amax(float amax) {
  return amax > 0.0f ? __fdiv_rn(2688.0f, amax) : 1.0f;
}

// This CTA's contiguous range of sub-tiles.
__device__ __forceinline__ void unit_range(int units, int& u0, int& u1) {
  u0 = static_cast<int>((static_cast<int64_t>(blockIdx.x) * units) / gridDim.x);
  u1 = static_cast<int>((static_cast<int64_t>(blockIdx.x + 1) * units) / gridDim.x);
}

// 14 warps: four of them share some SM sub-partition, whose 16 K registers
// then allow at most 128 a thread (checked once per device before the first
// launch).
// kSinglePass: the dynamic scale computed in this launch (phase A + grid
// barrier); a separate instance, so the static path carries none of it.
template <bool kSinglePass>
__global__ void __launch_bounds__(kThreads, 1)
    quantize_act_kernel(const __grid_constant__ CUtensorMap tmap_x,
                        const __grid_constant__ CUtensorMap tmap_l1, const QuantParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t l1_bytes = static_cast<uint32_t>(p.r) * 128u;
  uint8_t* xs = base;
  const int ns = p.stages;
  uint8_t* ls = xs + ns * kXTileBytes;
  float* inv_s = reinterpret_cast<float*>(ls + ns * l1_bytes);        // [K], touched columns
  float* gs_over_d = inv_s + p.K;                                     // [128] by E4M3 code
  uint8_t* cstage = reinterpret_cast<uint8_t*>(gs_over_d + 128);     // [kQuantWarps][32 rows][32 B]
  uint64_t* full = reinterpret_cast<uint64_t*>(cstage + kQuantWarps * 1024);
  uint64_t* qdone = full + kMaxStages;
  uint64_t* empty = qdone + kMaxStages;
  uint64_t* acc_full = empty + kMaxStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kblocks = p.K / kSubK;
  const bool has_lr = p.r > 0;
  const uint32_t tmem_cols = p.r <= 16 ? 32u : static_cast<uint32_t>(2 * p.r);
  int u0, u1;
  unit_range(p.units, u0, u1);
  // ring items: phase A (single-pass dynamic scale only), then phase B
  const int n_units = u1 - u0;
  const int phase_b0 = kSinglePass ? n_units : 0;   // first phase-B item
  const int n_items = phase_b0 + n_units;

  // Warp 0 sets up the barriers and issues the first ns loads as soon as
  // the other warps have issued their own set-up loads (s and gs): issued
  // after the x stream, those would wait behind it in the memory system and
  // hold the tables, and so the quantizers, back by microseconds.  The rest
  // of the CTA fills the RN(1/s) and RN(gs/scale) tables in the meantime.
  // Nobody else touches an mbarrier before the __syncthreads.  Global memory
  // only after the previous kernel on the stream is done.
  constexpr uint32_t kSetupBar = 6;  // named barrier: the set-up loads are issued
  pdl_launch_dependents();
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < ns; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&qdone[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tmap_x);
    if (has_lr) tma_prefetch_desc(&tmap_l1);
  }
  pdl_wait();
  const float gs_loaded = kSinglePass ? 1.0f : (p.gs_in ? *p.gs_in : tensor_scale_from_amax(*p.amax_src));
  if (warp == 0) named_bar_sync(kSetupBar, kThreads);
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < min(n_items, ns); ++i) {
      const int u = u0 + (i < n_units ? i : i - n_units);
      const bool l1 = has_lr && i >= phase_b0;
      const int rb = u / kblocks, kb = u % kblocks;
      mbar_arrive_expect_tx(&full[i], kXTileBytes + (l1 ? l1_bytes : 0u));
      tma_load_2d(xs + i * kXTileBytes, &tmap_x, &full[i], kb * kSubK, rb * kBM);
      if (l1) tma_load_2d(ls + i * l1_bytes, &tmap_l1, &full[i], kb * kSubK, 0);
    }
  }
  if (warp != 0) {
    // RN(1/s) for the columns of every sub-tile in [u0, u1): the whole K if
    // the range covers it, else per sub-tile (repeats write the same value).
    // Up to 8 columns a thread are loaded before the x stream goes out.
    const int t = threadIdx.x - 32, nt = kThreads - 32;
    const bool whole = u1 - u0 >= kblocks;
    const int ncols = whole ? p.K : (u1 - u0) * kSubK;
    auto column = [&](int j) { return whole ? j : ((u0 + j / kSubK) % kblocks) * kSubK + j % kSubK; };
    constexpr int kEarly = 8;
    float sv[kEarly];
#pragma unroll
    for (int e = 0; e < kEarly; ++e) {
      const int j = t + e * nt;
      sv[e] = (p.smooth_s && j < ncols) ? p.smooth_s[column(j)] : 1.0f;
    }
    named_bar_arrive(kSetupBar, kThreads);
#pragma unroll
    for (int e = 0; e < kEarly; ++e) {
      const int j = t + e * nt;
      if (j < ncols) inv_s[column(j)] = p.smooth_s ? __fdiv_rn(1.0f, sv[e]) : 1.0f;
    }
    for (int j = t + kEarly * nt; j < ncols; j += nt) {
      const int col = column(j);
      inv_s[col] = p.smooth_s ? __fdiv_rn(1.0f, p.smooth_s[col]) : 1.0f;
    }
  }
  if (warp == 1 && has_lr) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  // RN(gs / dec(sf)) for every finite E4M3 scale code (0 for the zero
  // scale): one IEEE division per code per CTA instead of one per group.
  // Single-pass dynamic scale: gs is known only after phase A.
  __shared__ uint32_t cta_amax_bits;
  __shared__ float gs_shared;
  __shared__ int grid_ok;
  if (threadIdx.x == 0) {
    cta_amax_bits = 0u;
    grid_ok = 1;
  }
  const float gs = gs_loaded;
  if (threadIdx.x < 128 && !kSinglePass) {
    const float d = e4m3_to_f32(threadIdx.x);
    gs_over_d[threadIdx.x] = (d == 0.0f || threadIdx.x == 127) ? 0.0f : __fdiv_rn(gs, d);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = has_lr ? *tmem_slot : 0u;

  if (warp == 0) {
    // ------------------------------------------------------- producer ----
    if (lane == 0) {
      int issued = min(n_items, ns);  // issued before the set-up sync
      for (int i = ns; i < n_items; ++i) {
        const int s = i % ns;
        const uint32_t ph = (i / ns) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, p.wait, kErrTimeoutEmpty)) break;
        const int u = u0 + (i < n_units ? i : i - n_units);
        const bool l1 = has_lr && i >= phase_b0;
        const int rb = u / kblocks, kb = u % kblocks;
        mbar_arrive_expect_tx(&full[s], kXTileBytes + (l1 ? l1_bytes : 0u));
        tma_load_2d(xs + s * kXTileBytes, &tmap_x, &full[s], kb * kSubK, rb * kBM);
        if (l1) tma_load_2d(ls + s * l1_bytes, &tmap_l1, &full[s], kb * kSubK, 0);
        issued = i + 1;
      }
      // never leave the CTA with a copy still landing in its shared memory
      for (int i = max(0, issued - ns); i < issued; ++i)
        mbar_wait(&full[i % ns], (i / ns) & 1, p.wait, kErrTimeoutDrain);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA ----
    if (has_lr && lane == 0) {
      const uint32_t idesc = idesc_f16(128, static_cast<uint32_t>(p.r), true);
      // descriptors of slot 0; a slot adds its byte offset >> 4 (shared
      // addresses stay below 256 KB).  No divisions in this loop: the tensor
      // pipe idles while the issuing thread computes.
      const uint64_t da0 = make_sdesc(smem_u32(xs), 16, 1024, kSwz128);
      const uint64_t db0 = make_sdesc(smem_u32(ls), 16, 1024, kSwz128);
      int seg = 0;             // segments started by this CTA
      bool first = true;       // first sub-tile of the current segment
      int s = phase_b0 % ns;   // ring slot of unit u's phase-B item
      uint32_t qd_par = 0;     // per slot: parity of its next qdone phase
      int kb = u0 % kblocks;   // 64-column block of unit u
      for (int u = u0; u < u1; ++u) {
        const int buf = seg & 1;
        if (first && seg >= 2 &&
            !mbar_wait(&acc_empty[buf], ((seg >> 1) - 1) & 1, p.wait, kErrTimeoutAcc))
          break;
        if (!mbar_wait(&qdone[s], (qd_par >> s) & 1u, p.wait, kErrTimeoutFull)) break;
        qd_par ^= 1u << s;
        tc_fence_after();
        const uint64_t da = da0 + ((static_cast<uint32_t>(s) * kXTileBytes) >> 4);
        const uint64_t db = db0 + ((static_cast<uint32_t>(s) * l1_bytes) >> 4);
        const uint32_t d = tmem + buf * static_cast<uint32_t>(p.r);
        umma_f16(d, da, db, idesc, first ? 0u : 1u);
#pragma unroll
        for (int kk = 1; kk < kSubK / 16; ++kk) umma_f16(d, da + 2 * kk, db + 2 * kk, idesc, 1u);
        umma_commit(&empty[s]);
        first = false;
        if (++s == ns) s = 0;
        const bool seg_end = (u + 1 == u1) || (kb + 1 == kblocks);  // the row block ends
        kb = kb + 1 == kblocks ? 0 : kb + 1;
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
    // Two warps per sub-tile: pair pq = qw / 2 takes ring items i = pq, pq + P,
    // pq + 2P, ... (P = ns / 2 pairs), item i in slot i % ns, so a pair owns
    // slots pq and pq + P and every barrier phase it waits on follows one it
    // consumed itself (a parity wait cannot tell a phase from the one two
    // before it).  Warp half h = qw % 2 takes rows 64h .. 64h + 63 of the
    // tile: lane l rows 64h + l and 64h + l + 32, each row's four 16-element
    // groups.  The pair agrees on every wait's verdict and meets before one
    // of its warps releases the slot.
    const size_t kbytes = static_cast<size_t>(p.K) / 2;
    const int npairs = ns / 2;
    const int pq = qw >> 1, hh = qw & 1;
    const bool active = pq < npairs;
    const uint32_t pair_bar = 2 + static_cast<uint32_t>(pq);  // named barrier of the pair (ids 2..5)
    int i = pq;              // ring item
    float gsq = gs;
    if constexpr (kSinglePass) {
      // phase A: max|x·inv_s| over this warp's half sub-tiles; each slot is
      // released as soon as both halves are read
      bool ok = true;
      float m8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (; active && i < phase_b0; i += npairs) {
        const int s = i % ns;
        // one verdict per pair: warps that disagree at the time limit must not split up
        const bool w_ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (i / ns) & 1, p.wait, kErrTimeoutFull));
        if (!named_bar_and(pair_bar, 64, w_ok)) {
          ok = false;
          break;
        }
        const float* isk = inv_s + ((u0 + i) % kblocks) * kSubK;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int row = 64 * hh + lane + 32 * j;
          const uint8_t* trow = xs + s * kXTileBytes + row * 128;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const uint4 v0 = *reinterpret_cast<const uint4*>(trow + (((2 * g) ^ (row & 7)) << 4));
            const uint4 v1 = *reinterpret_cast<const uint4*>(trow + (((2 * g + 1) ^ (row & 7)) << 4));
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            const float4* is4 = reinterpret_cast<const float4*>(isk + 16 * g);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float4 iv = is4[q];
              float a0, a1, a2, a3;
              mul_rn_x2(bf16lo(w[2 * q]), bf16hi(w[2 * q]), iv.x, iv.y, a0, a1);
              mul_rn_x2(bf16lo(w[2 * q + 1]), bf16hi(w[2 * q + 1]), iv.z, iv.w, a2, a3);
              m8[2 * q] = fmaxf(m8[2 * q], fmaxf(fabsf(a0), fabsf(a1)));
              m8[2 * q + 1] = fmaxf(m8[2 * q + 1], fmaxf(fabsf(a2), fabsf(a3)));
            }
          }
        }
        named_bar_sync(pair_bar, 64);
        if (hh == 0 && lane == 0) mbar_arrive(&empty[s]);
      }
      float am = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                       fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
      if (lane == 0) {
        atomicMax(&cta_amax_bits, __float_as_uint(am));  // non-negative floats order like their bits
        if (!ok) grid_ok = 0;
      }
      named_bar_sync(1, 32 * kQuantWarps);
      if (qw == 0 && lane == 0) {
        // one thread per CTA: fold the CTA's max in, then wait for every CTA
        atomicMax(&p.sync[1], cta_amax_bits);
        const bool skip = (p.fault & 2) && blockIdx.x == 0;  // test hook: this CTA never arrives
        const bool arrived = !skip && grid_arrive_wait(&p.sync[0], gridDim.x, p.wait);
        const float g = tensor_scale_from_amax(__uint_as_float(ld_acquire_gpu(&p.sync[1])));
        gs_shared = g;
        if (!arrived) grid_ok = 0;
        if (arrived && blockIdx.x == 0 && p.gs_copy) *p.gs_copy = g;
      }
      named_bar_sync(1, 32 * kQuantWarps);
      gsq = gs_shared;
      if (threadIdx.x - 64 < 128) {  // the RN(gs / dec(sf)) table, now that gs is known
        const uint32_t c = threadIdx.x - 64;
        const float d = e4m3_to_f32(c);
        gs_over_d[c] = (d == 0.0f || c == 127) ? 0.0f : __fdiv_rn(gsq, d);
      }
      const bool cta_ok = grid_ok != 0;
      named_bar_sync(1, 32 * kQuantWarps);
      if (!cta_ok) i = n_items;  // the barrier or a wait failed: quantize nothing
    } else {
      if (p.gs_copy && blockIdx.x == 0 && threadIdx.x == 64) *p.gs_copy = gs;
    }
    for (; active && i < n_items; i += npairs) {
      const int s = i % ns;
      const int u = u0 + i - phase_b0;
      const bool w_ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (i / ns) & 1, p.wait, kErrTimeoutFull));
      if (!named_bar_and(pair_bar, 64, w_ok)) break;
      const int rb = u / kblocks, kb = u % kblocks;
      const float* isk = inv_s + kb * kSubK;
      uint8_t* sfb = p.sf_out + (static_cast<size_t>(rb) * kblocks + kb) * 512 + lane * 16;
      uint8_t* stg = cstage + qw * 1024;  // this warp's 32 rows x 32 code bytes
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int row = 64 * hh + lane + 32 * j;
        uint8_t* trow = xs + s * kXTileBytes + row * 128;
        uint32_t codes[8];
        uint32_t sfw = 0;  // the row's four scale bytes
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint8_t* c0p = trow + (((2 * g) ^ (row & 7)) << 4);
          uint8_t* c1p = trow + (((2 * g + 1) ^ (row & 7)) << 4);
          const uint4 v0 = *reinterpret_cast<const uint4*>(c0p);
          const uint4 v1 = *reinterpret_cast<const uint4*>(c1p);
          const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
          float xh[16];
          const float4* is4 = reinterpret_cast<const float4*>(isk + 16 * g);
#pragma unroll
          for (int q = 0; q < 4; ++q) {  // x̂ = x·inv_s, two IEEE products per instruction
            const float4 iv = is4[q];
            mul_rn_x2(bf16lo(w[2 * q]), bf16hi(w[2 * q]), iv.x, iv.y, xh[4 * q], xh[4 * q + 1]);
            mul_rn_x2(bf16lo(w[2 * q + 1]), bf16hi(w[2 * q + 1]), iv.z, iv.w, xh[4 * q + 2], xh[4 * q + 3]);
          }
          // group max as a tree (max is exact, so the order does not matter)
          float m8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) m8[e] = fmaxf(fabsf(xh[e]), fabsf(xh[e + 8]));
#pragma unroll
          for (int e = 0; e < 4; ++e) m8[e] = fmaxf(m8[e], m8[e + 4]);
          const float amax = fmaxf(fmaxf(m8[0], m8[2]), fmaxf(m8[1], m8[3]));
          const float t = __fmul_rn(div6_rn(amax), gsq);
          const uint32_t sf = cvt_e4m3(t);
          const float inv = gs_over_d[sf & 127u];  // RN(gs / dec(sf)); 0 for a zero scale
          sfw |= sf << (8 * g);
          // cvt.rn.satfinite.e2m1x2 rounds ties to even and keeps the sign of
          // a value that rounds to zero (code 0x8), as the format requires;
          // the bit-exact tests hold it to that
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float q8[8];
#pragma unroll
            for (int e = 0; e < 8; e += 2) mul_rn_x2(xh[8 * h + e], xh[8 * h + e + 1], inv, inv, q8[e], q8[e + 1]);
            codes[2 * g + h] = cvt_e2m1x8(q8);
          }
          if (has_lr) {  // bf16(x̂) back over the tile, for the down-projection
            *reinterpret_cast<uint4*>(c0p) = make_uint4(pack_bf16x2(xh[0], xh[1]), pack_bf16x2(xh[2], xh[3]),
                                                        pack_bf16x2(xh[4], xh[5]), pack_bf16x2(xh[6], xh[7]));
            *reinterpret_cast<uint4*>(c1p) = make_uint4(pack_bf16x2(xh[8], xh[9]), pack_bf16x2(xh[10], xh[11]),
                                                        pack_bf16x2(xh[12], xh[13]), pack_bf16x2(xh[14], xh[15]));
          }
        }
        // the pass's 32 rows of 32 code bytes go out through shared memory,
        // so that each store writes whole 32-byte rows (16 per instruction)
        // instead of halves of 32 rows
        reinterpret_cast<uint4*>(stg + lane * 32)[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
        reinterpret_cast<uint4*>(stg + lane * 32)[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int rr = 16 * k + (lane >> 1);  // row of the pass; lane & 1: its half
          const int g2 = rb * kBM + 64 * hh + 32 * j + rr;
          const uint4 v = reinterpret_cast<const uint4*>(stg)[32 * k + lane];
          if (g2 < p.M)
            *reinterpret_cast<uint4*>(p.q_out + static_cast<size_t>(g2) * kbytes + kb * (kSubK / 2) +
                                      (lane & 1) * 16) = v;
        }
        __syncwarp();  // the next pass reuses the staging rows
        // the row's four scales: bytes (row % 32)·16 + (row / 32)·4 + g of the
        // 512-byte block; rows past M inside the last 128-row block hold
        // zero-filled x, so their scales are the zero padding the layout needs
        *reinterpret_cast<uint32_t*>(sfb + 4 * (2 * hh + j)) = sfw;
      }
      if (has_lr) fence_proxy_async_smem();
      named_bar_sync(pair_bar, 64);  // both halves done
      if (hh == 0 && lane == 0) mbar_arrive(has_lr ? &qdone[s] : &empty[s]);
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
  pdl_launch_dependents();
  pdl_wait();
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
// xl = 0 before the quantize kernel adds its partial sums (a row block's K
// range spans several CTAs), and the words the dynamic scale accumulates
// into (the single-pass grid barrier's counter and max, or the max pass's
// max); a kernel rather than memset nodes, so that programmatic dependent
// launch chains it to its neighbours.
__global__ void __launch_bounds__(256) clear_kernel(float4* __restrict__ p, size_t n4, uint32_t* __restrict__ words,
                                                    int nwords) {
  pdl_launch_dependents();
  pdl_wait();
  if (blockIdx.x == 0 && static_cast<int>(threadIdx.x) < nwords) words[threadIdx.x] = 0u;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    p[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
}

__global__ void act_scale_finalize_kernel(float* gs) {
  pdl_launch_dependents();
  pdl_wait();
  const float amax = __uint_as_float(*reinterpret_cast<unsigned*>(gs));
  *gs = tensor_scale_from_amax(amax);
}

}  // namespace

namespace {
constexpr size_t kSmemLimit = 227 * 1024 - 64;  // less the kernel's static shared words
size_t quantize_fixed_bytes(int64_t K) {
  return 1024 + static_cast<size_t>(K) * 4 + 128 * 4 + kQuantWarps * 1024 + 8 * (3 * kMaxStages + 4) + 16;
}
// Ring depth: as many sub-tiles as fit next to the RN(1/s) table, 2..8.
int quantize_stages(int64_t K, int r) {
  const size_t fixed = quantize_fixed_bytes(K);
  const size_t per = kXTileBytes + static_cast<size_t>(r) * 128;
  const int fit = fixed < kSmemLimit ? static_cast<int>((kSmemLimit - fixed) / per) : 0;
  return std::max(2, std::min(kMaxStages, fit)) & ~1;  // even: a warp pair owns two slots
}
}  // namespace

// Scratch of svdq_quantize_act_dynamic_noalloc: the grid-barrier counter and
// the max word of the single-pass dynamic scale, in a static device array
// instead of a caller's workspace.  Every device that loads the library
// holds it until the process exits; every call shares it.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];
static_assert(SVDQ_QUANTIZE_WORKSPACE_BYTES <= kNoallocScratchBytes, "the workspace must fit the array");

svdq_status noalloc_quantize_scratch(const LaunchCtx& ctx, uint32_t** out) {
  // its device address, looked up once per device and context with that
  // device current (host code cannot use the array's name as a device
  // pointer; a device reset makes a new context, where the array has a new
  // address)
  static std::mutex mu;
  static void* addr[64] = {};
  static unsigned long long ctx_of[64] = {};
  std::lock_guard<std::mutex> lk(mu);
  const int device = ctx.device;
  if (device < 0 || device >= 64) return fail(SVDQ_ERR_CUDA, "device index %d too large", device);
  if (!addr[device] || ctx_of[device] != ctx.ctx_id) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess)
      return fail(SVDQ_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    addr[device] = p;
    ctx_of[device] = ctx.ctx_id;
  }
  *out = static_cast<uint32_t*>(addr[device]);
  return SVDQ_OK;
}

size_t quantize_smem_bytes(int64_t K, int r) {
  return quantize_fixed_bytes(K) +
         static_cast<size_t>(quantize_stages(K, r)) * (kXTileBytes + static_cast<size_t>(r) * 128);
}

svdq_status launch_quantize_act(const LaunchCtx& ctx, const void* x, int64_t M, int64_t K,
                                int64_t ldx, const float* smooth_s, const void* L1t, int r,
                                const float* act_gscale, float* act_gscale_out, uint8_t* q_out,
                                uint8_t* sf_out, float* lora_out, uint32_t* grid_sync) {
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
  p.stages = quantize_stages(K, r);
  p.smooth_s = smooth_s;
  p.gs_in = act_gscale;
  const bool single_pass = !act_gscale && grid_sync;
  p.amax_src = (act_gscale || single_pass) ? nullptr : act_gscale_out;
  p.gs_copy = single_pass ? act_gscale_out
                          : ((act_gscale && act_gscale_out && act_gscale_out != act_gscale)
                                 ? act_gscale_out
                                 : nullptr);
  p.sync = single_pass ? grid_sync : nullptr;
  p.fault = ctx.fault_flags;
  p.q_out = q_out;
  p.sf_out = sf_out;
  p.lora_out = lora_out;
  p.wait = WaitCfg{ctx.timeout_ns, ctx.err_word};

  cudaStream_t st = ctx.stream;
  // lora_out is 16-byte aligned and M·r a multiple of 16; the dynamic scale's
  // words: the workspace (single pass) or act_gscale_out (max pass)
  uint32_t* words = single_pass ? grid_sync : (!act_gscale ? reinterpret_cast<uint32_t*>(act_gscale_out) : nullptr);
  const int nwords = single_pass ? 2 : (!act_gscale ? 1 : 0);
  if (r > 0 || nwords > 0) {
    const size_t n4 = static_cast<size_t>(M) * r / 4;
    const int blocks = static_cast<int>(
        std::max<size_t>(1, std::min<size_t>((n4 + 255) / 256, 2 * static_cast<size_t>(ctx.num_sms))));
    if (svdq_status e = launch_kernel(ctx, "clear_kernel", clear_kernel, dim3(blocks), dim3(256), 0,
                                      reinterpret_cast<float4*>(lora_out), n4, words, nwords))
      return e;
  }
  if (!single_pass && !act_gscale) {
    const int bx = static_cast<int>((K / 8 + 255) / 256);
    const int by = static_cast<int>(std::min<int64_t>(M, std::max(1, 4 * ctx.num_sms / bx)));
    if (svdq_status e = launch_kernel(ctx, "act_amax_kernel", act_amax_kernel, dim3(bx, by), dim3(256), 0,
                                      static_cast<const uint16_t*>(x), p.M, p.K, ldx, smooth_s,
                                      reinterpret_cast<unsigned*>(act_gscale_out)))
      return e;
  }
  const size_t smem = quantize_smem_bytes(K, r);
  {
    // four of the 14 warps share one SM sub-partition (16 K registers)
    static const bool regs_ok = [] {
      cudaFuncAttributes fa{};
      for (const void* fn : {reinterpret_cast<const void*>(quantize_act_kernel<false>),
                             reinterpret_cast<const void*>(quantize_act_kernel<true>)})
        if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess || fa.numRegs > 128) return false;
      return true;
    }();
    if (!regs_ok) return fail(SVDQ_ERR_CUDA, "quantize_act_kernel needs more than 128 registers a thread");
    const void* fn = single_pass ? reinterpret_cast<const void*>(quantize_act_kernel<true>)
                                 : reinterpret_cast<const void*>(quantize_act_kernel<false>);
    if (svdq_status e = set_smem_attr(ctx, fn, static_cast<int>(kSmemLimit))) return e;
  }
  const int grid = std::min(p.units, ctx.num_sms);
  if (single_pass) {
    // the CTAs meet at a grid barrier: all of them must be resident at once
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, quantize_act_kernel<true>, tx, tl, p);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return fail(SVDQ_ERR_CUDA, "quantize_act_kernel (cooperative): %s", cudaGetErrorString(e));
    }
    return SVDQ_OK;
  }
  if (svdq_status e = launch_kernel(ctx, "quantize_act_kernel", quantize_act_kernel<false>, dim3(grid),
                                    dim3(kThreads), smem, tx, tl, p))
    return e;
  if (!act_gscale) {
    if (svdq_status e = launch_kernel(ctx, "act_scale_finalize_kernel", act_scale_finalize_kernel, dim3(1),
                                      dim3(1), 0, act_gscale_out))
      return e;
  }
  return SVDQ_OK;
}

}  // namespace svdq
