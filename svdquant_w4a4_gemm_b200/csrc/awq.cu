// awq.cu — awq_w4a16_linear: int4-weight (group 64, fp16 scale and zero)
// by bf16-activation linear for M <= 8 rows, the bandwidth-bound modulation
// layers of the pages (ainews.surl.tw paragraph 2: "more sensitive modulation
// layers, or those limited by memory bandwidth, use AWQ W4A16").
//
// The kernel is bound by the weight stream (0.5 B/weight + 4 B per 64
// weights of scale and zero).  Dequantizing in registers with fp32 FMAs
// would cost M FMAs per weight on the CUDA cores (12+ us at M = 8 for a
// 3072 x 18432 layer, above the ~5 us HBM time), so the contraction runs on
// the tensor cores through mma.sync.m16n8k16 (bf16 in, fp32 accumulate), with
// the weights as the 16-row A operand taken straight from registers and the
// (tiny) activation as the B operand:
//   * per lane, one 8-byte load per weight row and 64-wide group: 16 nibbles;
//     nibble pairs (j, j+4) become bf16 pairs 128+q with one LOP3, and one
//     bf16x2 subtract of (128+z) gives the exact integers q − z;
//   * each group's partial product (4 MMAs, k = 64) is scaled by its fp16
//     scale in fp32, so the integer weights stay exact;
//   * x̂ = x·(1/a) is split into bf16 hi + lo parts (two B columns) so the
//     activation keeps ~16 significant bits; for M <= 4 hi and lo share one
//     8-column B tile, for 4 < M <= 8 they take two.
// The k order inside an MMA is permuted to match the nibble pairs; the B
// fragments are built once per CTA in shared memory in that order, while
// the CTA's first weight loads are already in flight.  A CTA owns 4 weight
// tiles of 16 rows; two warps share each tile, one per half of K, each
// streaming its rows with a double-buffered register prefetch; the halves
// are combined through shared memory in a fixed order.
#include "internal.h"
#include "ptx.cuh"

namespace svdq {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kTilesPerCta = 4;       // 16-row weight tiles per CTA
constexpr int kSplit = kWarps / kTilesPerCta;  // warps (K ranges) per tile
constexpr int kBatch = 4;             // groups per prefetch batch (double-buffered)

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t bsub2(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&a),
                             *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One prefetch batch of a lane: per group, 8 bytes of each of its two rows
// and the two rows' fp16 scale and zero.
struct Batch {
  uint2 wa[kBatch], wb[kBatch];
  __half2 sc[kBatch], zz[kBatch];  // (row a, row b)
};

__device__ __forceinline__ void load_batch(Batch& b, int G0, int Gend, const uint2* qa,
                                           const uint2* qb, const __half* sa, const __half* sb,
                                           const __half* za, const __half* zb) {
#pragma unroll
  for (int u = 0; u < kBatch; ++u) {
    const int G = G0 + u;
    if (G < Gend) {
      b.wa[u] = __ldcs(qa + G * 4);  // 4 lanes x 8 B = one 32-byte sector per row and group
      b.wb[u] = __ldcs(qb + G * 4);
      b.sc[u] = __halves2half2(sa[G], sb[G]);
      b.zz[u] = __halves2half2(za[G], zb[G]);
    }
  }
}

template <int NT>
__device__ __forceinline__ void compute_batch(const Batch& b, int G0, int Gend, const uint2* bfrag,
                                              int lane, float (&acc)[NT][4]) {
#pragma unroll
  for (int u = 0; u < kBatch; ++u) {
    const int G = G0 + u;
    if (G >= Gend) break;
    const float2 scf = __half22float2(b.sc[u]);
    const float2 zf = __half22float2(b.zz[u]);
    const uint32_t za2 = bf16x2_bits(128.0f + zf.x, 128.0f + zf.x);
    const uint32_t zb2 = bf16x2_bits(128.0f + zf.y, 128.0f + zf.y);
    float cg[NT][4] = {};
    const uint2* bf = bfrag + static_cast<size_t>(G) * 4 * 32 * NT;
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const uint32_t Wa = w ? b.wa[u].y : b.wa[u].x;
      const uint32_t Wb = w ? b.wb[u].y : b.wb[u].x;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int s = 2 * w + h;
        const uint32_t a0 = bsub2(((Wa >> (8 * h)) & 0x000F000Fu) | 0x43004300u, za2);
        const uint32_t a2 = bsub2(((Wa >> (8 * h + 4)) & 0x000F000Fu) | 0x43004300u, za2);
        const uint32_t a1 = bsub2(((Wb >> (8 * h)) & 0x000F000Fu) | 0x43004300u, zb2);
        const uint32_t a3 = bsub2(((Wb >> (8 * h + 4)) & 0x000F000Fu) | 0x43004300u, zb2);
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          const uint2 bb = bf[(s * 32 + lane) * NT + j];
          mma_bf16(cg[j], a0, a1, a2, a3, bb.x, bb.y);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      acc[j][0] = fmaf(cg[j][0], scf.x, acc[j][0]);
      acc[j][1] = fmaf(cg[j][1], scf.x, acc[j][1]);
      acc[j][2] = fmaf(cg[j][2], scf.y, acc[j][2]);
      acc[j][3] = fmaf(cg[j][3], scf.y, acc[j][3]);
    }
  }
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 2)
    awq_w4a16_kernel(const uint16_t* __restrict__ x, int M, int K,
                     const float* __restrict__ ainv, const uint32_t* __restrict__ qw,
                     const __half* __restrict__ scales, const __half* __restrict__ zeros,
                     const uint16_t* __restrict__ bias, int N, uint16_t* __restrict__ y) {
  extern __shared__ uint2 bfrag[];  // [K/64][4 steps][32 lanes][NT]; then the K-split partials
  const int groups = K / 64;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int ntiles = N / 16;
  const int tile = blockIdx.x * kTilesPerCta + (warp % kTilesPerCta);
  const int part = warp / kTilesPerCta;                  // which K range
  const int Gbeg = (groups * part) / kSplit, Gend = (groups * (part + 1)) / kSplit;
  const bool active = tile < ntiles;
  const int n_a = (active ? tile : 0) * 16 + g, n_b = n_a + 8;
  const uint2* qa = reinterpret_cast<const uint2*>(qw + static_cast<size_t>(n_a) * (K / 8)) + t;
  const uint2* qb = reinterpret_cast<const uint2*>(qw + static_cast<size_t>(n_b) * (K / 8)) + t;
  const __half* sa = scales + static_cast<size_t>(n_a) * groups;
  const __half* sb = scales + static_cast<size_t>(n_b) * groups;
  const __half* za = zeros + static_cast<size_t>(n_a) * groups;
  const __half* zb = zeros + static_cast<size_t>(n_b) * groups;

  // the first weight batch is in flight while the B table is built
  Batch cur, nxt;
  if (active) load_batch(cur, Gbeg, Gend, qa, qb, sa, sb, za, zb);

  // ---- B fragments: column c of tile j holds token m's hi or lo part ----
  // One item = (group G, lane, tile j): its 4 steps need x̂ at the 16
  // contiguous k = 64G + 16·t .. +16 of one token, read with vector loads.
#pragma unroll 2
  for (int e = threadIdx.x; e < groups * 32 * NT; e += kThreads) {
    const int j = e % NT;
    const int ln = (e / NT) & 31;
    const int G = e / NT / 32;
    const int gg = ln >> 2, tt = ln & 3;
    const int m = NT == 1 ? (gg & 3) : gg;
    const int hl = NT == 1 ? (gg >> 2) : j;
    const int k0 = 64 * G + 16 * tt;
    float v[16];
    if (m < M) {
      const uint4* xv = reinterpret_cast<const uint4*>(x + static_cast<size_t>(m) * K + k0);
      const uint4 u0 = xv[0], u1 = xv[1];
      const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
      float av[16];
      if (ainv) {
        const float4* a4 = reinterpret_cast<const float4*>(ainv + k0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 a = a4[q];
          av[4 * q] = a.x; av[4 * q + 1] = a.y; av[4 * q + 2] = a.z; av[4 * q + 3] = a.w;
        }
      }
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        float xv1 = __uint_as_float((q & 1) ? (w[q >> 1] & 0xFFFF0000u) : (w[q >> 1] << 16));
        if (ainv) xv1 = __fmul_rn(xv1, av[q]);
        const float hi = __bfloat162float(__float2bfloat16_rn(xv1));
        v[q] = hl == 0 ? hi : __fsub_rn(xv1, hi);
      }
    } else {
#pragma unroll
      for (int q = 0; q < 16; ++q) v[q] = 0.0f;
    }
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int kb = 8 * (s >> 1) + 2 * (s & 1);  // offset of slot 2t within the 16
      bfrag[((G * 4 + s) * 32 + ln) * NT + j] =
          make_uint2(bf16x2_bits(v[kb], v[kb + 4]), bf16x2_bits(v[kb + 1], v[kb + 5]));
    }
  }
  __syncthreads();

  float acc[NT][4] = {};
  if (active) {
    for (int G0 = Gbeg; G0 < Gend; G0 += kBatch) {
      if (G0 + kBatch < Gend) load_batch(nxt, G0 + kBatch, Gend, qa, qb, sa, sb, za, zb);
      compute_batch<NT>(cur, G0, Gend, bfrag, lane, acc);
      cur = nxt;
    }
  }
  // ---- combine the K ranges: parts 1.. leave partials in shared memory ----
  float* part_s = reinterpret_cast<float*>(bfrag + static_cast<size_t>(groups) * 4 * 32 * NT);
  if (part > 0) {
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q)
        part_s[(((part - 1) * kTilesPerCta + (warp % kTilesPerCta)) * 32 + lane) * 4 * NT + 4 * j + q] =
            acc[j][q];
  }
  __syncthreads();
  if (part > 0 || !active) return;
#pragma unroll
  for (int pp = 1; pp < kSplit; ++pp)
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q)
        acc[j][q] += part_s[(((pp - 1) * kTilesPerCta + warp) * 32 + lane) * 4 * NT + 4 * j + q];

  // c0,c1: row n_a, columns 2t, 2t+1; c2,c3: row n_b, same columns
  float r0, r1, r2, r3;
  bool store;
  if (NT == 1) {
    // columns 0-3 hold the hi parts of tokens 0-3, columns 4-7 the lo parts
    r0 = acc[0][0] + __shfl_xor_sync(0xffffffffu, acc[0][0], 2);
    r1 = acc[0][1] + __shfl_xor_sync(0xffffffffu, acc[0][1], 2);
    r2 = acc[0][2] + __shfl_xor_sync(0xffffffffu, acc[0][2], 2);
    r3 = acc[0][3] + __shfl_xor_sync(0xffffffffu, acc[0][3], 2);
    store = t < 2;
  } else {
    r0 = acc[0][0] + acc[NT - 1][0];
    r1 = acc[0][1] + acc[NT - 1][1];
    r2 = acc[0][2] + acc[NT - 1][2];
    r3 = acc[0][3] + acc[NT - 1][3];
    store = true;
  }
  if (store) {
    const float ba = bias ? __uint_as_float(static_cast<uint32_t>(bias[n_a]) << 16) : 0.0f;
    const float bb = bias ? __uint_as_float(static_cast<uint32_t>(bias[n_b]) << 16) : 0.0f;
    const float out[2][2] = {{r0, r2}, {r1, r3}};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int m = 2 * t + i;
      if (m < M) {
        __nv_bfloat16 va = __float2bfloat16_rn(out[i][0] + ba);
        __nv_bfloat16 vb = __float2bfloat16_rn(out[i][1] + bb);
        y[static_cast<size_t>(m) * N + n_a] = *reinterpret_cast<uint16_t*>(&va);
        y[static_cast<size_t>(m) * N + n_b] = *reinterpret_cast<uint16_t*>(&vb);
      }
    }
  }
}

}  // namespace

svdq_status launch_awq_w4a16(const LaunchCtx& ctx, const void* x, int64_t M, int64_t K,
                             const float* act_scale_inv, const uint32_t* qweight,
                             const void* scales, const void* zeros, const void* bias, int64_t N,
                             void* y) {
  const int ntiles = static_cast<int>(N / 16);
  const int grid = (ntiles + kTilesPerCta - 1) / kTilesPerCta;
  const int nt = M <= 4 ? 1 : 2;
  const size_t smem = static_cast<size_t>(K) * 16 * nt +
                      static_cast<size_t>(kSplit - 1) * kTilesPerCta * 32 * 4 * nt * sizeof(float);
  auto kern = nt == 1 ? awq_w4a16_kernel<1> : awq_w4a16_kernel<2>;
  if (svdq_status e = set_smem_attr(ctx, reinterpret_cast<const void*>(kern), 227 * 1024)) return e;
  kern<<<grid, kThreads, smem, ctx.stream>>>(
      static_cast<const uint16_t*>(x), static_cast<int>(M), static_cast<int>(K), act_scale_inv,
      qweight, static_cast<const __half*>(scales), static_cast<const __half*>(zeros),
      static_cast<const uint16_t*>(bias), static_cast<int>(N), static_cast<uint16_t*>(y));
  return check_launch("awq_w4a16_kernel");
}

}  // namespace svdq
