// awq.cu — awq_w4a16_linear: int4-weight (group 64, fp16 scale and zero)
// by bf16-activation linear for M <= 8 rows, the bandwidth-bound modulation
// layers of the pages (ainews.surl.tw, paragraph 2: the layers that are
// precision-sensitive, like the modulation layers, or memory-bound keep int4
// weights with 16-bit activations, AWQ W4A16).
//
// The op is bound by the weight stream (0.5 B/weight + 4 B per 64 weights of
// scale and zero).  Dequantizing in registers with fp32 FMAs would cost M
// FMAs per weight on the CUDA cores (12+ us at M = 8 for a 3072 x 18432
// layer, above the ~5 us HBM time), so the contraction runs on the tensor
// cores through mma.sync.m16n8k16 (bf16 in, fp32 accumulate), with the
// weights as the 16-row A operand taken straight from registers and the
// (tiny) activation as the B operand:
//   * nibble pairs (j, j+4) of a weight word become bf16 pairs 128+q with one
//     LOP3, and one bf16x2 subtract of (128+z) gives the exact integers q − z;
//   * each group's partial product (4 MMAs, k = 64) is scaled by its fp16
//     scale in fp32, so the integer weights stay exact;
//   * x̂ = x·(1/a) is split into bf16 hi + lo parts (two B columns) so the
//     activation keeps ~16 significant bits; for M <= 4 hi and lo share one
//     8-column B tile, for 4 < M <= 8 they take two.
// The k order inside an MMA is permuted to match the nibble pairs, and the
// activation fragments use the same order.  Two kernels: the streaming
// kernel (below, the default) stages 16-row weight strips through a
// shared-memory ring with TMA; the register-streaming kernel (first) takes
// the shapes the streaming kernel does not (scales or zeros not 16-byte
// aligned, K not a multiple of 256 or above 3072, more than 16 strips per
// SM).  It keeps the B fragments in shared memory, built once per CTA while
// its first weight loads are in flight; a CTA owns 4 weight tiles of 16
// rows, two warps per tile (one per half of K) each streaming its rows with a
// double-buffered register prefetch of 8 bytes per row and group, the halves
// combined through shared memory in a fixed order.
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
  pdl_launch_dependents();
  pdl_wait();  // global memory only after the previous kernel on the stream is done
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

// ---------------------------------------------------------------------------
// Streaming kernel (the default): one persistent CTA per SM takes a contiguous
// range of 16-row weight strips.  A producer thread first copies the inverse
// smoothing scales (1/a, K floats) into shared memory, then each strip with
// one 3-D TMA copy (the strip's K/256 chunks of 128 bytes x 16 rows, chunk
// major, 128-byte swizzle) and two bulk copies (its scales and zeros) into a
// ring of shared-memory slots as deep as shared memory allows (7 slots, ~190
// KB in flight per SM at K = 3072, so a CTA's whole share of the HBM stream
// is requested at once).  The weight stream goes out only after the
// consumers have issued their loads of x, which would otherwise wait behind
// it in the memory system.  In a slot, 128-byte
// line c·16 + r holds chunk c of row r with its 16-byte units XOR-ed by r mod
// 8, so ldmatrix reads of the same unit of 8 rows hit 8 distinct bank groups.
//
// Twelve consumer warps split K: warp w always takes the same K/12 range, so
// its activation fragments (x̂ = x·(1/a), bf16 hi and lo) are built once, in
// registers, from one batch of loads of x (a warp with fewer than GMAX
// groups runs the missing ones on zero fragments).  Per 64-wide group a lane takes
// one ldmatrix.x4 (rows g and g+8, both 32-wide halves: 4 words of 8
// nibbles), turns nibble pairs (i, i+4) into bf16 pairs 128 + q with one
// LOP3 and into exact q − z with one bf16x2 subtract, and issues 4
// mma.sync.m16n8k16 per B tile, in the k order the nibble pairs give (the
// activation fragments use the same order), the groups' accumulation chains
// interleaved; each group's partial product is scaled by its fp16 scale in
// fp32.  A warp adds its hi and lo columns, leaves its K range's partial sums
// of the strip (16 rows x up to 8 tokens) in one of two shared-memory buffers
// and goes on to the next strip; a reducer warp sums the twelve partials in a
// fixed order, adds the bias and stores y as bf16, then hands the buffer back.
constexpr int kSWarps = 12;                      // consumer warps (K ranges)
constexpr int kSProducer = kSWarps;              // warp index of the producer
constexpr int kSReducer = kSWarps + 1;           // warp index of the reducer
constexpr int kSThreads = 32 * (kSWarps + 2);
constexpr int kSRows = 16;                       // weight rows per strip
constexpr int kSMaxStrips = 16;                  // strips per CTA whose bias is staged
constexpr int kSPartFloats = kSWarps * 32 * 4;   // one strip's partials: [warp][lane][4]

struct StreamLayout {
  int chunks;         // 128-byte chunks of a weight row (K / 256)
  int qbytes;         // 16 rows, chunk-major
  int sbytes;         // scales (or zeros) of the strip: 16 rows x K/64 fp16
  int slot;           // qbytes + 2 sbytes rounded up to 1 KB (the swizzle atom)
  int abytes;         // 1/a: K floats, rounded up to 1 KB
  int stages;
  // shared memory from the 1 KB-aligned base: partials [2][kSPartFloats],
  // 1/a, the ring, then bias (kSMaxStrips x 16 bf16) and the mbarriers
  __host__ __device__ int ring_offset() const { return (2 * kSPartFloats * 4 + abytes + 1023) / 1024 * 1024; }
  __host__ __device__ int tail_offset() const { return ring_offset() + stages * slot; }
  __host__ __device__ int bytes() const { return tail_offset() + kSMaxStrips * kSRows * 2 + 8 * (2 * stages + 5); }
};

__host__ __device__ inline StreamLayout stream_layout(int K) {
  StreamLayout L;
  L.chunks = K / 256;
  L.qbytes = kSRows * L.chunks * 128;
  L.sbytes = kSRows * (K / 64) * 2;
  L.slot = (L.qbytes + 2 * L.sbytes + 1023) / 1024 * 1024;
  L.abytes = (K * 4 + 1023) / 1024 * 1024;
  L.stages = 8;
  while (L.stages > 2 && 1024 + L.bytes() > 227 * 1024) --L.stages;
  return L;
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                            uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// NT: B tiles of 8 columns (1: hi and lo of up to 4 tokens in one tile; 2: hi
// tile and lo tile of up to 8 tokens).  GMAX: 64-wide groups per warp.
template <int NT, int GMAX>
__global__ void __launch_bounds__(kSThreads, 1)
    awq_w4a16_stream_kernel(const __grid_constant__ CUtensorMap tmap_q, const uint16_t* __restrict__ x, int M, int K,
                            const float* __restrict__ ainv, const __half* __restrict__ scales,
                            const __half* __restrict__ zeros, const uint16_t* __restrict__ bias, int N,
                            uint16_t* __restrict__ y, WaitCfg wait) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int groups = K / 64;
  const StreamLayout L = stream_layout(K);
  float* part = reinterpret_cast<float*>(base);                            // [2][kSPartFloats]
  float* ainv_s = reinterpret_cast<float*>(base + 2 * kSPartFloats * 4);  // [K]
  uint8_t* ring = base + L.ring_offset();                                  // 1 KB aligned
  uint16_t* bias_s = reinterpret_cast<uint16_t*>(base + L.tail_offset());  // [kSMaxStrips * 16]
  uint64_t* full = reinterpret_cast<uint64_t*>(base + L.tail_offset() + kSMaxStrips * kSRows * 2);
  uint64_t* empty = full + L.stages;
  uint64_t* red_full = empty + L.stages;   // [2] the consumers' partials of a strip are in the buffer
  uint64_t* red_empty = red_full + 2;      // [2] the reducer has read the buffer
  uint64_t* abar = red_empty + 2;          // 1/a has landed
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nstrips = N / kSRows;
  const int s0 = static_cast<int>((static_cast<int64_t>(blockIdx.x) * nstrips) / gridDim.x);
  const int s1 = static_cast<int>((static_cast<int64_t>(blockIdx.x + 1) * nstrips) / gridDim.x);
  const int nmine = s1 - s0;

  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < L.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kSWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&red_full[b], kSWarps);
      mbar_init(&red_empty[b], 1);
    }
    mbar_init(abar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();  // global memory only after the previous kernel on the stream is done

  // the consumers' loads of x go out before the weight stream: issued after
  // it, they would wait behind it in the memory system and hold every
  // consumer back by microseconds
  constexpr uint32_t kXIssued = 1;                       // named barrier
  constexpr uint32_t kXIssuedThreads = 32 * (kSWarps + 1);  // consumers + producer
  if (warp == kSProducer) {
    // ------------------------------------------------------ producer ----
    // lane 0: 1/a, then (once x is requested) the strips into the ring as
    // slots come free
    if (lane == 0) {
      tma_prefetch_desc(&tmap_q);
      if (ainv) {
        mbar_arrive_expect_tx(abar, static_cast<uint32_t>(K * 4));
        bulk_load(ainv_s, ainv, static_cast<uint32_t>(K * 4), abar);
      }
    }
    named_bar_sync(kXIssued, kXIssuedThreads);
    if (lane == 0) {
      const uint32_t bytes = static_cast<uint32_t>(L.qbytes + 2 * L.sbytes);
      int issued = 0;
      for (int i = 0; i < nmine; ++i) {
        const int s = i % L.stages;
        if (i >= L.stages && !mbar_wait(&empty[s], ((i / L.stages) & 1) ^ 1, wait, kErrTimeoutEmpty)) break;
        uint8_t* slot = ring + s * L.slot;
        const size_t n0 = static_cast<size_t>(s0 + i) * kSRows;
        mbar_arrive_expect_tx(&full[s], bytes);
        tma_load_3d(slot, &tmap_q, &full[s], 0, static_cast<int32_t>(n0), 0);
        bulk_load(slot + L.qbytes, scales + n0 * groups, static_cast<uint32_t>(L.sbytes), &full[s]);
        bulk_load(slot + L.qbytes + L.sbytes, zeros + n0 * groups, static_cast<uint32_t>(L.sbytes), &full[s]);
        issued = i + 1;
      }
      // never leave the CTA with a copy still landing in its shared memory
      if (ainv) mbar_wait(abar, 0, wait, kErrTimeoutDrain);
      for (int i = issued > L.stages ? issued - L.stages : 0; i < issued; ++i)
        mbar_wait(&full[i % L.stages], (i / L.stages) & 1, wait, kErrTimeoutDrain);
    }
    return;
  }

  if (warp == kSReducer) {
    // ------------------------------------------------------- reducer ----
    // the bias of this CTA's rows into shared memory, once
    for (int e = lane; e < nmine * kSRows; e += 32)
      bias_s[e] = bias ? bias[static_cast<size_t>(s0) * kSRows + e] : static_cast<uint16_t>(0);
    __syncwarp();
    // lane L: rows L/4 and L/4 + 8 of the strip, tokens 2·(L % 4) and +1
    const int r0 = lane >> 2, m0 = 2 * (lane & 3);
    for (int i = 0; i < nmine; ++i) {
      const int b = i & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&red_full[b], (i >> 1) & 1, wait, kErrTimeoutFull))) break;
      const float4* pb = reinterpret_cast<const float4*>(part + b * kSPartFloats) + lane;
      float4 v = pb[0];
#pragma unroll
      for (int w = 1; w < kSWarps; ++w) {
        const float4 u = pb[w * 32];
        v.x += u.x;
        v.y += u.y;
        v.z += u.z;
        v.w += u.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&red_empty[b]);  // the buffer may be refilled
      const float ba = __uint_as_float(static_cast<uint32_t>(bias_s[i * kSRows + r0]) << 16);
      const float bb = __uint_as_float(static_cast<uint32_t>(bias_s[i * kSRows + r0 + 8]) << 16);
      const size_t n = static_cast<size_t>(s0 + i) * kSRows + r0;
      const float o[4] = {v.x + ba, v.y + ba, v.z + bb, v.w + bb};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int m = m0 + (e & 1);
        if (m < M) {
          const __nv_bfloat16 h = __float2bfloat16_rn(o[e]);
          y[static_cast<size_t>(m) * N + n + 8 * (e >> 1)] = *reinterpret_cast<const uint16_t*>(&h);
        }
      }
    }
    return;
  }

  // ---------------------------------------------------------- consumers ----
  const int g = lane >> 2, t = lane & 3;
  const int gb = (groups * warp) / kSWarps, ge = (groups * (warp + 1)) / kSWarps;  // this warp's groups
  // B fragments: per group, half s (32 of its 64 k), MMA j of the half, tile
  // nt: {b0, b1} = x̂ at k = base + 2j + {0, 4} and base + 2j + {1, 5}, base =
  // 64G + 32s + 8t, token column g (NT = 1: token g & 3, hi for g < 4, lo for
  // g >= 4; NT = 2: token g, tile 0 hi, tile 1 lo).  A warp with fewer than
  // GMAX groups runs the missing ones on group 0's weights with zero
  // fragments: they add exact zeros, and the strip loop needs no branch.
  uint32_t bf[GMAX][2][2][NT][2];
  {
    const int m = NT == 1 ? (g & 3) : g;
    uint4 xr[GMAX][2];
#pragma unroll
    for (int gi = 0; gi < GMAX; ++gi)
#pragma unroll
      for (int s = 0; s < 2; ++s) {  // all loads of x first: one round trip
        const bool v = m < M && gb + gi < ge;
        const size_t off = v ? static_cast<size_t>(m) * K + 64 * (gb + gi) + 32 * s + 8 * t : 0;
        xr[gi][s] = __ldg(reinterpret_cast<const uint4*>(x + off));
        if (!v) xr[gi][s] = make_uint4(0u, 0u, 0u, 0u);
      }
    named_bar_arrive(kXIssued, kXIssuedThreads);
    if (ainv) __all_sync(0xffffffffu, mbar_wait(abar, 0, wait, kErrTimeoutFull));
#pragma unroll
    for (int gi = 0; gi < GMAX; ++gi)
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const int k0 = 64 * (gb + gi) + 32 * s + 8 * t;
        const uint32_t w8[4] = {xr[gi][s].x, xr[gi][s].y, xr[gi][s].z, xr[gi][s].w};
        float xv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          xv[e] = __uint_as_float((e & 1) ? (w8[e >> 1] & 0xFFFF0000u) : (w8[e >> 1] << 16));
        if (ainv && gb + gi < ge) {
          const float4 a0 = *reinterpret_cast<const float4*>(ainv_s + k0);
          const float4 a1 = *reinterpret_cast<const float4*>(ainv_s + k0 + 4);
          const float a8[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) xv[e] = __fmul_rn(xv[e], a8[e]);
        }
        float hi[8], lo[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          hi[e] = __bfloat162float(__float2bfloat16_rn(xv[e]));
          lo[e] = __fsub_rn(xv[e], hi[e]);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const bool use_lo = NT == 1 ? (g >= 4) : (nt == 1);
            const float* v = use_lo ? lo : hi;
            bf[gi][s][j][nt][0] = bf16x2_bits(v[2 * j], v[2 * j + 4]);
            bf[gi][s][j][nt][1] = bf16x2_bits(v[2 * j + 1], v[2 * j + 5]);
          }
      }
  }
  // Per group, the byte offsets in a slot of this lane's ldmatrix row address
  // (lane L reads row (L & 7) + 8·((L >> 3) & 1) of half L >> 4 of the group:
  // 16-byte unit u = 2·(G % 4) + half of chunk G / 4, at line (G / 4)·16 +
  // row, unit u XOR (row % 8)) and of row g's scale in the scale block (row
  // g + 8 lies 8·K/64 scales further; the zeros follow the scales).
  uint32_t qoff[GMAX], soff[GMAX];
  {
    const int lrow = (lane & 7) + 8 * ((lane >> 3) & 1), lhalf = lane >> 4;
#pragma unroll
    for (int gi = 0; gi < GMAX; ++gi) {
      const int G = gb + gi < ge ? gb + gi : 0;
      qoff[gi] = static_cast<uint32_t>((G >> 2) * (kSRows * 128) + lrow * 128 +
                                       (((2 * (G & 3) + lhalf) ^ (lrow & 7)) << 4));
      soff[gi] = static_cast<uint32_t>(g * groups + G) * 2;
    }
  }
  const uint32_t ring_u32 = smem_u32(ring);
  const int row8 = 8 * groups;  // scales between rows g and g + 8
  int s = 0;
  uint32_t phase = 0;
  for (int i = 0; i < nmine; ++i) {
    const bool got = __all_sync(0xffffffffu, mbar_wait(&full[s], phase, wait, kErrTimeoutFull));
    float acc[NT][4] = {};
    if (got) {
      const uint32_t qs = ring_u32 + static_cast<uint32_t>(s * L.slot);
      const uint8_t* sblk = ring + s * L.slot + L.qbytes;
      // CH groups at a time (all of them with one B tile; two with two B
      // tiles, which leaves registers for the fragments): their words and
      // scales first, then the MMAs with the groups' accumulation chains
      // interleaved
      constexpr int CH = NT == 1 ? GMAX : 2;
#pragma unroll
      for (int c0 = 0; c0 < GMAX; c0 += CH) {
        uint32_t R[CH][4];  // (row g, half 0), (row g+8, half 0), (row g, half 1), (row g+8, half 1)
        uint32_t za2[CH], zb2[CH];
        float sca[CH], scb[CH];
#pragma unroll
        for (int ci = 0; ci < CH; ++ci) {
          if (c0 + ci >= GMAX) continue;
          ldmatrix_x4(qs + qoff[c0 + ci], R[ci][0], R[ci][1], R[ci][2], R[ci][3]);
          const __half* sc = reinterpret_cast<const __half*>(sblk + soff[c0 + ci]);
          const __half* zz = reinterpret_cast<const __half*>(sblk + L.sbytes + soff[c0 + ci]);
          sca[ci] = __half2float(sc[0]);
          scb[ci] = __half2float(sc[row8]);
          const float za = 128.0f + __half2float(zz[0]), zb = 128.0f + __half2float(zz[row8]);
          za2[ci] = bf16x2_bits(za, za);
          zb2[ci] = bf16x2_bits(zb, zb);
        }
        float cg[CH][NT][4] = {};
#pragma unroll
        for (int hs = 0; hs < 2; ++hs)
#pragma unroll
          for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int ci = 0; ci < CH; ++ci) {
              if (c0 + ci >= GMAX) continue;
              const uint32_t Wa = R[ci][2 * hs], Wb = R[ci][2 * hs + 1];
              const uint32_t a0 = bsub2(((Wa >> (8 * j)) & 0x000F000Fu) | 0x43004300u, za2[ci]);
              const uint32_t a2 = bsub2(((Wa >> (8 * j + 4)) & 0x000F000Fu) | 0x43004300u, za2[ci]);
              const uint32_t a1 = bsub2(((Wb >> (8 * j)) & 0x000F000Fu) | 0x43004300u, zb2[ci]);
              const uint32_t a3 = bsub2(((Wb >> (8 * j + 4)) & 0x000F000Fu) | 0x43004300u, zb2[ci]);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                mma_bf16(cg[ci][nt], a0, a1, a2, a3, bf[c0 + ci][hs][j][nt][0], bf[c0 + ci][hs][j][nt][1]);
            }
#pragma unroll
        for (int ci = 0; ci < CH; ++ci) {
          if (c0 + ci >= GMAX) continue;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            acc[nt][0] = fmaf(cg[ci][nt][0], sca[ci], acc[nt][0]);
            acc[nt][1] = fmaf(cg[ci][nt][1], sca[ci], acc[nt][1]);
            acc[nt][2] = fmaf(cg[ci][nt][2], scb[ci], acc[nt][2]);
            acc[nt][3] = fmaf(cg[ci][nt][3], scb[ci], acc[nt][3]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);  // this warp has read the strip
    // hi + lo: one B tile holds hi in columns 0-3 and lo in 4-7 (lane + 2),
    // two tiles hold them in tiles 0 and 1; lane L then holds rows L/4 and
    // L/4 + 8, tokens 2·(L % 4) and +1 (one tile: lanes L % 4 < 2 only)
    float v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      v[q] = NT == 1 ? acc[0][q] + __shfl_down_sync(0xffffffffu, acc[0][q], 2) : acc[0][q] + acc[NT - 1][q];
    // into buffer i % 2 once the reducer has read its previous strip
    const int b = i & 1;
    if (i >= 2) __all_sync(0xffffffffu, mbar_wait(&red_empty[b], ((i >> 1) - 1) & 1, wait, kErrTimeoutEmpty));
    reinterpret_cast<float4*>(part + b * kSPartFloats)[warp * 32 + lane] = make_float4(v[0], v[1], v[2], v[3]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&red_full[b]);
    if (++s == L.stages) {
      s = 0;
      phase ^= 1;
    }
  }
}

}  // namespace

namespace {
template <int NT, int GMAX>
svdq_status launch_stream(const LaunchCtx& ctx, const void* x, int M, int K, const float* ainv,
                          const uint32_t* qweight, const void* scales, const void* zeros,
                          const void* bias, int N, void* y) {
  const StreamLayout L = stream_layout(K);
  const size_t smem = 1024 + static_cast<size_t>(L.bytes());
  auto kern = awq_w4a16_stream_kernel<NT, GMAX>;
  if (svdq_status e = set_smem_attr(ctx, reinterpret_cast<const void*>(kern), static_cast<int>(smem))) return e;
  // weights as bytes: (128 bytes of a chunk, row, chunk), box = one strip
  CUtensorMap tq{};
  if (!make_tmap_3d_u8(&tq, qweight, 128, static_cast<uint64_t>(N), static_cast<uint64_t>(L.chunks),
                       static_cast<uint64_t>(K) / 2, 128, 128, kSRows, static_cast<uint32_t>(L.chunks), true))
    return SVDQ_ERR_CUDA;
  const int grid = std::min(N / kSRows, ctx.num_sms);
  return launch_kernel(ctx, "awq_w4a16_stream_kernel", kern, dim3(grid), dim3(kSThreads), smem, tq,
                       static_cast<const uint16_t*>(x), M, K, ainv, static_cast<const __half*>(scales),
                       static_cast<const __half*>(zeros), static_cast<const uint16_t*>(bias), N,
                       static_cast<uint16_t*>(y), WaitCfg{ctx.timeout_ns, ctx.err_word});
}
}  // namespace

svdq_status launch_awq_w4a16(const LaunchCtx& ctx_in, const void* x, int64_t M, int64_t K,
                             const float* act_scale_inv, const uint32_t* qweight,
                             const void* scales, const void* zeros, const void* bias, int64_t N,
                             void* y) {
  // With two B tiles (M > 4) the streaming kernel measured ~1.2 us slower on
  // B200 when launched with programmatic dependent launch than in plain
  // stream order (with one tile it is ~1 us faster), so those launches go
  // in plain order; the results are the same either way.
  LaunchCtx ctx = ctx_in;
  if (M > 4) ctx.pdl = 0;
  // the streaming kernel: K/64 groups split over 12 warps, each holding the
  // activation fragments of at most 4 groups in registers; the TMA box takes
  // whole 128-byte chunks of a row (K % 256 == 0), the bulk copies of scales,
  // zeros and 1/a and the 16-byte loads of x need 16-byte alignment, and
  // shared memory holds the bias of at most kSMaxStrips strips
  const int groups = static_cast<int>(K / 64);
  const int gpw = (groups + kSWarps - 1) / kSWarps;
  const bool aligned = ((reinterpret_cast<uintptr_t>(scales) | reinterpret_cast<uintptr_t>(zeros) |
                         reinterpret_cast<uintptr_t>(act_scale_inv) | reinterpret_cast<uintptr_t>(x)) & 15) == 0;
  const int64_t strips_per_cta = (N / kSRows + ctx.num_sms - 1) / ctx.num_sms;
  if (aligned && K % 256 == 0 && gpw <= 4 && strips_per_cta <= kSMaxStrips) {
    const int m = static_cast<int>(M), k = static_cast<int>(K), n = static_cast<int>(N);
    if (M <= 4) {
      if (gpw <= 2) return launch_stream<1, 2>(ctx, x, m, k, act_scale_inv, qweight, scales, zeros, bias, n, y);
      if (gpw <= 3) return launch_stream<1, 3>(ctx, x, m, k, act_scale_inv, qweight, scales, zeros, bias, n, y);
      return launch_stream<1, 4>(ctx, x, m, k, act_scale_inv, qweight, scales, zeros, bias, n, y);
    }
    if (gpw <= 2) return launch_stream<2, 2>(ctx, x, m, k, act_scale_inv, qweight, scales, zeros, bias, n, y);
    if (gpw <= 3) return launch_stream<2, 3>(ctx, x, m, k, act_scale_inv, qweight, scales, zeros, bias, n, y);
    return launch_stream<2, 4>(ctx, x, m, k, act_scale_inv, qweight, scales, zeros, bias, n, y);
  }
  // otherwise the register-streaming kernel above (B fragments in shared memory)
  const int ntiles = static_cast<int>(N / 16);
  const int grid = (ntiles + kTilesPerCta - 1) / kTilesPerCta;
  const int nt = M <= 4 ? 1 : 2;
  const size_t smem = static_cast<size_t>(K) * 16 * nt +
                      static_cast<size_t>(kSplit - 1) * kTilesPerCta * 32 * 4 * nt * sizeof(float);
  auto kern = nt == 1 ? awq_w4a16_kernel<1> : awq_w4a16_kernel<2>;
  if (svdq_status e = set_smem_attr(ctx, reinterpret_cast<const void*>(kern), 227 * 1024)) return e;
  return launch_kernel(ctx, "awq_w4a16_kernel", kern, dim3(grid), dim3(kThreads), smem,
                       static_cast<const uint16_t*>(x), static_cast<int>(M), static_cast<int>(K), act_scale_inv,
                       qweight, static_cast<const __half*>(scales), static_cast<const __half*>(zeros),
                       static_cast<const uint16_t*>(bias), static_cast<int>(N), static_cast<uint16_t*>(y));
}

}  // namespace svdq
