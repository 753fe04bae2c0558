// gemm_common.cuh — what the two W4A4 GEMM kernels (one SM per 128-row
// tile in gemm.cu, SM pairs per 256-row tile in gemm_pair.cu) share: the
// launch parameters, the staging of block scales into tensor memory, the
// in-place conversion of the low-rank activation slice into its MMA operand,
// and the epilogue arithmetic of one 64-column output box.
#pragma once

#include "internal.h"
#include "ptx.cuh"

namespace svdq {

constexpr int kGemmBKBytes = 128;  // 256 FP4 elements per FP4 step and row

struct GemmParams {
  int M, N, K, r;
  int tiles_n, tiles;     // output tiles along N, total
  const uint8_t* sf_a;
  const uint8_t* sf_w;
  const float* gs_a;
  const float* gs_w;
  const uint16_t* bias;   // [N] or null
  int n_part;             // split output: columns per part (tmap_y, tmap_y1, tmap_y2); 0 = one output
  int fault;              // test hook: 1 = the first ring slot never fills
  WaitCfg wait;
};

// GELU, tanh form, in fp32: 0.5·v·(1 + tanh(√(2/π)·(v + 0.044715·v³))).
// The hardware tanh keeps the activation off the epilogue's critical path
// (one MUFU op per element); its ~2^-11 relative error is below the bf16
// rounding of the output that follows.
__device__ __forceinline__ float gelu_tanh(float v) {
  const float u = 0.7978845608028654f * fmaf(0.044715f * v, v * v, v);
  const float h = 0.5f * v;
  return fmaf(h, tanh_approx(u), h);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// One FP4 step's block scales from shared memory into a TMEM scale region
// (called by one warp per 32-lane quadrant; every quadrant holds the same
// copy).  Lane l, column j of a region holds the four E4M3 scales (one
// 64-K block) of tile row 32j + l, the order the block-scaled MMA reads.
// SFA: columns 4kk + j = bytes [4j, 4j + 4) of line `lane` of 128x4 block
// kk (`a_valid` false: zeros, for a row block past the operand).  SFB:
// columns 16 + (BN/32)kk + j hold tile row 32j + lane.  BN = 192 spans two
// 128-row scale blocks: n0 % 128 == 0 takes the line of block 0 (rows
// 0-127) then words 0-1 of block 1 (rows 128-191); n0 % 128 == 64 (hi64)
// takes words 2-3 of block 0 (rows 0-63) then the line of block 1 (rows
// 64-191).
template <int BN>
__device__ __forceinline__ void stage_scales(const uint8_t* sfa_slot, const uint8_t* sfb_slot, int lane,
                                             bool hi64, bool a_valid, uint32_t sfr) {
  const uint8_t* sa = sfa_slot + lane * 16;
  const uint8_t* sb = sfb_slot + lane * 16;
  uint32_t va[16];
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    uint4 u = make_uint4(0u, 0u, 0u, 0u);
    if (a_valid) u = *reinterpret_cast<const uint4*>(sa + kk * 512);
    va[4 * kk] = u.x;
    va[4 * kk + 1] = u.y;
    va[4 * kk + 2] = u.z;
    va[4 * kk + 3] = u.w;
  }
  tmem_st_32x32b_x16(sfr, va);
  if constexpr (BN == 128) {
    uint32_t vb[16];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint4 x = *reinterpret_cast<const uint4*>(sb + kk * 512);
      vb[4 * kk] = x.x;
      vb[4 * kk + 1] = x.y;
      vb[4 * kk + 2] = x.z;
      vb[4 * kk + 3] = x.w;
    }
    tmem_st_32x32b_x16(sfr + 16, vb);
  } else {
    static_assert(BN == 192, "scale staging covers BN = 128 and 192");
    uint32_t vb[24];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint4 x = *reinterpret_cast<const uint4*>(sb + (hi64 ? 2048 : 0) + kk * 512);
      const uint2 y = *reinterpret_cast<const uint2*>(sb + (hi64 ? 8 : 2048) + kk * 512);
      const uint32_t lo[6] = {x.x, x.y, x.z, x.w, y.x, y.y};
      const uint32_t hi[6] = {y.x, y.y, x.x, x.y, x.z, x.w};
#pragma unroll
      for (int j = 0; j < 6; ++j) vb[6 * kk + j] = hi64 ? hi[j] : lo[j];
    }
    const uint32_t v16[16] = {vb[0], vb[1], vb[2],  vb[3],  vb[4],  vb[5],  vb[6],  vb[7],
                              vb[8], vb[9], vb[10], vb[11], vb[12], vb[13], vb[14], vb[15]};
    const uint32_t v8[8] = {vb[16], vb[17], vb[18], vb[19], vb[20], vb[21], vb[22], vb[23]};
    tmem_st_32x32b_x16(sfr + 16, v16);
    tmem_st_32x32b_x8(sfr + 32, v8);
  }
}

// The low-rank A operand of one tile row, in place: the row's 32 fp32 values
// of the xl slice sit unswizzled in its own 128 bytes; they are replaced by
// 32 columns of hi = bf16(xl·gprod) and 32 of lo = bf16(xl·gprod − hi)
// (gprod = gs_a·gs_w), in the 128-byte swizzled K-major layout.
__device__ __forceinline__ void lowrank_operand_row(uint8_t* arow, int row, float gprod) {
  float w[32];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 u = *reinterpret_cast<const float4*>(arow + 16 * q);
    w[4 * q] = u.x;
    w[4 * q + 1] = u.y;
    w[4 * q + 2] = u.z;
    w[4 * q + 3] = u.w;
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {  // chunk q: hi of columns 8q..8q+7; chunk 4+q: their lo
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float t0 = __fmul_rn(w[8 * q + 2 * e], gprod);
      const float t1 = __fmul_rn(w[8 * q + 2 * e + 1], gprod);
      const float h0 = __bfloat162float(__float2bfloat16_rn(t0));
      const float h1 = __bfloat162float(__float2bfloat16_rn(t1));
      hw[e] = pack_bf16x2(h0, h1);
      lw[e] = pack_bf16x2(__fsub_rn(t0, h0), __fsub_rn(t1, h1));
    }
    *reinterpret_cast<uint4*>(arow + ((q ^ (row & 7)) << 4)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4*>(arow + (((4 + q) ^ (row & 7)) << 4)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
}

// Columns [64j, 64j + 64) of this warp's 32 accumulator rows: TMEM ->
// α·acc + bias [-> GELU] -> 32 packed bf16 pairs.
template <bool kGelu>
__device__ __forceinline__ void epilogue_box(uint32_t taddr_box, const uint16_t* bias_box, float alpha,
                                             uint32_t (&packed)[32]) {
#pragma unroll
  for (int c = 0; c < 4; c += 2) {  // 16-column chunks, two per load pair
    uint32_t v0[16], v1[16];
    tmem_ld_32x32b_x16(taddr_box + c * 16, v0);
    tmem_ld_32x32b_x16(taddr_box + (c + 1) * 16, v1);
    tmem_ld_wait();
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const uint32_t* av = u ? v1 : v0;
      const uint4* b4 = reinterpret_cast<const uint4*>(bias_box + (c + u) * 16);
      const uint4 bb0 = b4[0], bb1 = b4[1];
      const uint32_t bw[8] = {bb0.x, bb0.y, bb0.z, bb0.w, bb1.x, bb1.y, bb1.z, bb1.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float lo = __fadd_rn(__fmul_rn(__uint_as_float(av[2 * e]), alpha), __uint_as_float(bw[e] << 16));
        float hi = __fadd_rn(__fmul_rn(__uint_as_float(av[2 * e + 1]), alpha),
                             __uint_as_float(bw[e] & 0xFFFF0000u));
        if (kGelu) {
          lo = gelu_tanh(lo);
          hi = gelu_tanh(hi);
        }
        packed[(c + u) * 8 + e] = pack_bf16x2(lo, hi);
      }
    }
  }
}

// The packed 32 x 64 bf16 box into its shared-memory staging area (128-byte
// swizzle; row `lane` of the box is this lane's row).
__device__ __forceinline__ void write_box(uint8_t* brow, int lane, const uint32_t (&packed)[32]) {
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *reinterpret_cast<uint4*>(brow + ((q ^ (lane & 7)) << 4)) =
        make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
}

// Which output tensor map and column a tile at output column n0 goes to
// (a tile never straddles two parts of a split output).
__device__ __forceinline__ const CUtensorMap* output_map(const GemmParams& p, int n0, const CUtensorMap* y,
                                                         const CUtensorMap* y1, const CUtensorMap* y2,
                                                         int& ycol) {
  ycol = n0;
  if (!p.n_part) return y;
  const int part = n0 / p.n_part;
  ycol = n0 - part * p.n_part;
  return part == 0 ? y : (part == 1 ? y1 : y2);
}

// The SM-pair kernel (gemm_pair.cu): 256 x bn output tiles (bn = 128 or
// 192 dividing N / parts).  The B and L2ᵀ tensor maps have bn / 2-row boxes.
svdq_status launch_w4a4_gemm_pair(const LaunchCtx& ctx, const CUtensorMap& ta, const CUtensorMap& tb,
                                  const CUtensorMap& tl, const CUtensorMap& ty, const CUtensorMap& tr,
                                  const CUtensorMap& ty1, const CUtensorMap& ty2, GemmParams p, int bn,
                                  int activation);

}  // namespace svdq
