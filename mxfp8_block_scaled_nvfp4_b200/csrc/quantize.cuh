// HBM-bound elementwise kernels: tensor amax, NVFP4 / MXFP8 quantize,
// dequantize and the standalone scale re-layout.
//
// Work mapping.  A tensor [rows, K] is viewed as a flat sequence of
// "half-blocks" of 8 consecutive elements (K % 16 == 0, so a 16-element NVFP4
// block is two adjacent half-blocks of the same row, and a 32-element MXFP8
// block four).  Lane l of a warp takes half-block base + l, so one warp load
// instruction reads 32 x 16 contiguous bytes (bf16 / fp16), the block amax
// is two (NVFP4) or three (MXFP8) xor-shuffles, and each lane stores one
// packed uint32 of eight e2m1 codes (NVFP4) or two of e4m3 codes (MXFP8):
// 128 or 256 contiguous bytes per warp store.  Scales are written by the
// first lane of each block, directly at their LINEAR or 128x4-tile offset.
// Grids are persistent (a multiple of the SM count); each warp processes
// kUnroll x 32 half-blocks per iteration to keep several loads in flight.
#pragma once

#include "common.cuh"

namespace nvfp4 {

constexpr int kEwThreads = 256;
constexpr int kUnroll = 4;

// ---------------------------------------------------------------------------
// a1: g = max |x| of up to 4 tensors in one launch, each atomically combined
// into its own output (which the host zeroes).  Each thread keeps 4
// independent 16-byte loads in flight per iteration.
// ---------------------------------------------------------------------------
constexpr int kAmaxSegs = 4;

struct AmaxSegs {
  const void* x[kAmaxSegs];
  int64_t n[kAmaxSegs];
  float* out[kAmaxSegs];
  uint32_t count;
};

template <typename T>
__global__ void __launch_bounds__(kEwThreads) k_amax(const __grid_constant__ AmaxSegs a) {
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t nthr = (int64_t)gridDim.x * blockDim.x;
  __shared__ float red[kEwThreads / 32];
  for (uint32_t sgi = 0; sgi < a.count; ++sgi) {
    const T* x = static_cast<const T*>(a.x[sgi]);
    const int64_t n = a.n[sgi];
    const int64_t nvec = n / 8;
    float m = 0.0f;
    // raw 16-byte words of 4 vectors, the next 4 in flight while these are
    // reduced (zero words past the end reduce to 0)
    constexpr int W = sizeof(T) == 4 ? 2 : 1;
    uint4 nxt[4][W];
    auto load4 = [&](int64_t i0) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int64_t j = i0 + k * nthr;
        const uint4* q = reinterpret_cast<const uint4*>(x + j * 8);
#pragma unroll
        for (int w = 0; w < W; ++w) nxt[k][w] = j < nvec ? __ldg(q + w) : make_uint4(0, 0, 0, 0);
      }
    };
    load4(tid);
    for (int64_t i = tid; i < nvec; i += 4 * nthr) {
      uint4 cur[4][W];
#pragma unroll
      for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int w = 0; w < W; ++w) cur[k][w] = nxt[k][w];
      load4(i + 4 * nthr);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float v[8];
        unpack8<T>(cur[k][0], cur[k][W - 1], v);
#pragma unroll
        for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(v[e]));
      }
    }
    for (int64_t i = nvec * 8 + tid; i < n; i += nthr) m = fmaxf(m, fabsf(Elem<T>::to_f(x[i])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
      m = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      // non-negative floats order like their bit patterns
      if (threadIdx.x == 0) atomicMax(reinterpret_cast<unsigned int*>(a.out[sgi]), __float_as_uint(m));
    }
    __syncthreads();  // red is reused by the next tensor
  }
}

// ---------------------------------------------------------------------------
// Shared pieces of the quantizers
// ---------------------------------------------------------------------------
struct ScaleOut {
  uint8_t* p;
  uint32_t blocks_per_row;  // K / group
  uint32_t Cp;              // padded columns (swizzled) = ceil4(blocks_per_row)
  bool swizzled;
  FastDiv bpr;              // division by blocks_per_row (block index -> row)
  __host__ void init(uint8_t* scales, uint32_t bpr_, bool swz) {
    p = scales;
    blocks_per_row = bpr_;
    Cp = (bpr_ + 3u) / 4u * 4u;
    swizzled = swz;
    bpr.init(bpr_ ? bpr_ : 1u);
  }
  // byte offset of block `block` (flat index over [rows, blocks_per_row])
  __device__ __forceinline__ uint32_t offset(uint32_t block) const {
    if (!swizzled) return block;
    const uint32_t r = bpr.div(block), c = block - r * blocks_per_row;
    return swizzled_offset(r, c, Cp);
  }
  __device__ __forceinline__ void store(uint32_t block, uint32_t byte) const { p[offset(block)] = (uint8_t)byte; }
};

// Zero the padding bytes of a 128x4-tile scale buffer: rows [rows, Rp) and
// columns [bpr, Cp) ("mlx 0.30.7.2 -> 0.30.7.6" diff, page 8, qqmm_utils.h,
// pad_and_swizzle_scales: out-of-bounds values must be zero).
__device__ __forceinline__ void zero_scale_padding(const ScaleOut& so, uint32_t rows) {
  if (!so.swizzled) return;
  const uint32_t Rp = (rows + 127u) & ~127u;
  const uint32_t tid = blockIdx.x * blockDim.x + threadIdx.x, nthr = gridDim.x * blockDim.x;
  const uint32_t n1 = (Rp - rows) * so.Cp;
  for (uint32_t i = tid; i < n1; i += nthr) {
    uint32_t r = rows + i / so.Cp, c = i % so.Cp;
    so.p[swizzled_offset(r, c, so.Cp)] = 0;
  }
  const uint32_t pc = so.Cp - so.blocks_per_row;
  if (pc == 0) return;
  const uint32_t n2 = rows * pc;
  for (uint32_t i = tid; i < n2; i += nthr) {
    uint32_t r = i / pc, c = so.blocks_per_row + i % pc;
    so.p[swizzled_offset(r, c, so.Cp)] = 0;
  }
}

// ---------------------------------------------------------------------------
// f4: stochastic rounding of the NVFP4 codes.  The pages reserve it
// ("mlx 0.30.7.2 -> 0.30.7.6" diff, page 7, fp_quantize_rowwise<..., USE_SR>
// with rbits "reserved for future use"); this library's reading: the block
// scale as in the round-to-nearest path, each scaled value t to one of its
// two e2m1 neighbours lo <= |t| <= hi, up iff b * 2^-8 < (|t| - lo) / (hi -
// lo) for 8 random bits b.  As the pages pass one 32-bit rbits word to each
// 4-value conversion, element i of the flat [rows, K] array takes byte i % 4
// of word i / 4, and word w is output w % 4 of Philox4x32-10 (Salmon,
// Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC
// 2011) at counter (w / 4 as 64 bits, 0, 0), key (seed).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint64_t p0 = (uint64_t)0xD2511F53u * c.x, p1 = (uint64_t)0xCD9E8D57u * c.z;  // one wide multiply each
    c = make_uint4((uint32_t)(p1 >> 32) ^ c.y ^ k0, (uint32_t)p1, (uint32_t)(p0 >> 32) ^ c.w ^ k1, (uint32_t)p0);
  }
  return c;
}

// e2m1 code of t with stochastic rounding by the random byte r (sign kept,
// saturating at 6), without branches: the grid has spacing 0.5 on [0, 2),
// 1 on [2, 4) and 2 on [4, 6), so pos = (|t| - base) / spacing is exact in
// fp32, floor(pos) indexes the lower neighbour and pos - floor(pos) is the
// exact position between the two neighbours.
__device__ __forceinline__ uint32_t e2m1_sr(float t, uint32_t r) {
  const float a = fabsf(t);
  const bool i0 = a < 2.0f, i1 = a < 4.0f;
  const float base = i0 ? 0.0f : (i1 ? 2.0f : 4.0f);
  const float inv_gap = i0 ? 2.0f : (i1 ? 1.0f : 0.5f);
  const uint32_t code0 = i0 ? 0u : (i1 ? 4u : 6u);
  const float pos = (a - base) * inv_gap;
  const float fl = floorf(pos);
  const float frac = pos - fl;
  const float u = (float)r * 0x1p-8f;
  uint32_t m = code0 + (uint32_t)fl + (u < frac ? 1u : 0u);
  m = a >= 6.0f ? 7u : m;
  return (signbit(t) ? 8u : 0u) | m;
}

// ---------------------------------------------------------------------------
// a2-a4: NVFP4 quantize of up to kMaxSegs tensors in one launch (the raw
// qqmm quantizes both operands, "mlx 0.30.7.2 -> 0.30.7.6" diff, page 8,
// ops.cpp qqmm; one launch over both keeps every SM busy on what would be
// two short launches).  Per 16-block: E = 2688 / g (1 without g);
//   s = e4m3_rne_satfinite((amax / 6) * E);  q_i = e2m1(x_i * (E / f8(s)))
// ("mlx 0.30.7.2 -> 0.30.7.6" diff, page 7, fp_quantize_rowwise), zero
// codes for a block whose scale decodes to 0.
//
// A lane quantizes whole 16-element blocks (K % 16 == 0: a block never
// leaves its row): one 32-byte load (bf16 / fp16; two for fp32, 256-bit
// vector loads when every input is 32-byte aligned), the block maximum in
// registers, one scale, two code words in one 8-byte store (a warp writes
// 256 contiguous bytes).  Work unit: 32 x kBlkU consecutive blocks of one
// tensor (one warp iteration); units of all tensors form one sequence, warp
// w takes units w, w + nwarps, ..., and the loads of its next unit are in
// flight while it computes the current one.  Scale bytes of 4 consecutive
// blocks go out as one 32-bit store where they are contiguous (LINEAR
// layout, or 4 blocks of one row starting at a multiple of 4 in the tile
// layout); other scales are stored byte by byte.  E / f8(s) comes from a
// per-CTA table of those IEEE quotients (0 <= s <= 0x7E).
// ---------------------------------------------------------------------------
constexpr int kMaxSegs = 4;
constexpr int kBlkU = 2;                          // blocks per lane per unit
constexpr uint32_t kUnitBlk = 32u * kBlkU;        // blocks per unit

struct QuantSeg {
  const void* x;
  const float* g;
  uint32_t* codes;
  ScaleOut so;
  uint32_t rows;
  uint32_t n_blk;       // 16-element blocks
  uint32_t first_unit;  // index of the segment's first unit in the launch's sequence
};

struct QuantSegs {
  QuantSeg s[kMaxSegs];
  uint32_t count;
  uint32_t units;  // all units of all segments
  uint64_t seed;   // stochastic rounding only
};

// Raw bytes of one 16-element block: 32 (2-byte types) or 64 (fp32).
template <typename T>
struct RawBlk {
  uint4 w[sizeof(T) == 4 ? 4 : 2];
};

template <bool V8>
__device__ __forceinline__ void ld32(const void* p, uint4& a, uint4& b) {
  if constexpr (V8) {
    asm volatile("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
                 : "l"(p));
  } else {
    const uint4* q = static_cast<const uint4*>(p);
    a = __ldg(q);
    b = __ldg(q + 1);
  }
}

template <typename T, bool V8>
__device__ __forceinline__ void load_blk(const T* p, RawBlk<T>& r) {
  ld32<V8>(p, r.w[0], r.w[1]);
  if constexpr (sizeof(T) == 4) ld32<V8>(reinterpret_cast<const uint8_t*>(p) + 32, r.w[2], r.w[3]);
}

template <typename T>
__device__ __forceinline__ void unpack16(const RawBlk<T>& r, float (&v)[16]) {
  float lo[8], hi[8];
  if constexpr (sizeof(T) == 4) {
    unpack8<T>(r.w[0], r.w[1], lo);
    unpack8<T>(r.w[2], r.w[3], hi);
  } else {
    unpack8<T>(r.w[0], r.w[0], lo);
    unpack8<T>(r.w[1], r.w[1], hi);
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    v[j] = lo[j];
    v[8 + j] = hi[j];
  }
}

__device__ __forceinline__ uint32_t seg_of(const QuantSegs& q, uint32_t unit) {
  uint32_t i = 0;
#pragma unroll
  for (int j = 1; j < kMaxSegs; ++j)
    if ((uint32_t)j < q.count && unit >= q.s[j].first_unit) i = (uint32_t)j;
  return i;
}

template <typename T, bool V8>
__device__ __forceinline__ void load_unit(const QuantSegs& q, uint32_t unit, uint32_t lane, RawBlk<T> (&r)[kBlkU]) {
  if (unit >= q.units) return;
  const QuantSeg& sg = q.s[seg_of(q, unit)];
  const uint32_t base = (unit - sg.first_unit) * kUnitBlk;
  const T* x = static_cast<const T*>(sg.x);
#pragma unroll
  for (int u = 0; u < kBlkU; ++u) {
    const uint32_t b = base + (uint32_t)u * 32u + lane;
    if (b < sg.n_blk) {
      load_blk<T, V8>(x + (size_t)b * 16, r[u]);
    } else {
#pragma unroll
      for (int i = 0; i < (int)(sizeof(r[u].w) / 16); ++i) r[u].w[i] = make_uint4(0, 0, 0, 0);
    }
  }
}

// Scale byte s of this lane's block b, 4 consecutive blocks per 32-bit
// store where possible.  All lanes call it.
__device__ __forceinline__ void store_scales(const ScaleOut& so, uint32_t b, uint32_t n_blk, uint32_t s,
                                             uint32_t lane) {
  const uint32_t s1 = __shfl_down_sync(0xffffffffu, s, 1);
  const uint32_t s2 = __shfl_down_sync(0xffffffffu, s, 2);
  const uint32_t s3 = __shfl_down_sync(0xffffffffu, s, 3);
  // lane % 4 == 0 owns blocks b0 .. b0 + 3 (b0 a multiple of 4)
  const uint32_t b0 = b & ~3u;
  bool packed = b0 + 4u <= n_blk;  // all four blocks exist
  uint32_t off = b0;
  if (so.swizzled) {
    const uint32_t r = so.bpr.div(b0), c = b0 - r * so.blocks_per_row;
    packed = packed && (c & 3u) == 0 && c + 4u <= so.blocks_per_row;
    off = swizzled_offset(r, c, so.Cp);
  }
  if (packed) {
    if ((lane & 3u) == 0) *reinterpret_cast<uint32_t*>(so.p + off) = __byte_perm(s | (s1 << 8), s2 | (s3 << 8), 0x5410);
  } else if (b < n_blk) {
    so.store(b, s);
  }
}

// e2m1 codes of v[i] * k for 8 values, each product rounded to fp32.
__device__ __forceinline__ uint32_t scaled_e2m1x8_at(const float (&v)[16], int o, float k) {
  float h[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) h[j] = v[o + j];
  return scaled_e2m1x8(h, k);
}

template <typename T, bool SR = false, bool V8 = false>
__global__ void __launch_bounds__(kEwThreads) k_nvfp4_quantize(const __grid_constant__ QuantSegs q) {
  __shared__ float ktab[kMaxSegs][128];
  __shared__ float etab[kMaxSegs];
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  RawBlk<T> nxt[kBlkU];
  load_unit<T, V8>(q, warp, lane, nxt);  // the first unit's loads before the table
  for (uint32_t i = threadIdx.x; i < q.count * 128u; i += blockDim.x) {
    const QuantSeg& sg = q.s[i >> 7];
    const float E = sg.g ? kGlobalEncode / __ldg(sg.g) : 1.0f;
    const float fs = e4m3_to_f32(i & 127u);
    ktab[i >> 7][i & 127u] = fs != 0.0f ? E / fs : 0.0f;
    if ((i & 127u) == 0) etab[i >> 7] = E;
  }
  __syncthreads();
  for (uint32_t unit = warp; unit < q.units; unit += nwarps) {
    RawBlk<T> cur[kBlkU];
#pragma unroll
    for (int u = 0; u < kBlkU; ++u) cur[u] = nxt[u];
    load_unit<T, V8>(q, unit + nwarps, lane, nxt);  // next unit's loads in flight during this one
    const uint32_t si = seg_of(q, unit);
    const QuantSeg& sg = q.s[si];
    const uint32_t base = (unit - sg.first_unit) * kUnitBlk;
    const float E = etab[si];
    const float* kt = ktab[si];
#pragma unroll
    for (int u = 0; u < kBlkU; ++u) {
      const uint32_t b = base + (uint32_t)u * 32u + lane;
      float v[16];
      unpack16<T>(cur[u], v);
      float a = 0.0f;
#pragma unroll
      for (int j = 0; j < 16; ++j) a = fmaxf(a, fabsf(v[j]));
      float t = a / kE2M1Max;
      t = t * E;
      const uint32_t s = f32_to_e4m3(t);
      uint2 w = make_uint2(0u, 0u);
      if constexpr (SR) {
        // the block's 16 random bytes: the four outputs of the generator at
        // counter b (elements 4i..4i+3 from output i, byte j for element
        // 4i+j); every lane calls it, outside the branches
        const uint4 r4 = philox4x32_10(make_uint4(b, 0u, 0u, 0u), (uint32_t)q.seed, (uint32_t)(q.seed >> 32));
        if (s != 0u) {
          const float k = kt[s];
          const uint32_t rw[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            w.x |= e2m1_sr(v[j] * k, (rw[j >> 2] >> (8 * (j & 3))) & 0xFFu) << (4 * j);
            w.y |= e2m1_sr(v[8 + j] * k, (rw[2 + (j >> 2)] >> (8 * (j & 3))) & 0xFFu) << (4 * j);
          }
        }
      } else {
        if (s != 0u) {  // f8(s) != 0
          const float k = kt[s];
          w.x = scaled_e2m1x8_at(v, 0, k);
          w.y = scaled_e2m1x8_at(v, 8, k);
        }
      }
      if (b < sg.n_blk) reinterpret_cast<uint2*>(sg.codes)[b] = w;
      store_scales(sg.so, b, sg.n_blk, s, lane);
    }
  }
  for (uint32_t i = 0; i < q.count; ++i) zero_scale_padding(q.s[i].so, q.s[i].rows);
}

// ---------------------------------------------------------------------------
// f1: column-wise NVFP4 quantize ("mlx 0.30.7.2 -> 0.30.7.6" diff, page 7,
// fp_quantize.cu, fp_quantize_columnwise: an M-major [M, K] input quantized
// along K): x [R, C] row-major is quantized as x^T [C, R] along R, with the
// same per-block arithmetic as k_nvfp4_quantize.  Codes [C, R/8], scales
// [C, R/16] (LINEAR or 128x4 tiles).  This is what the backward pass of the
// dense matmul needs for w^T and x^T and for the transposed upstream
// gradient.
//
// CTA tile: 128 rows x 64 columns of x, staged in shared memory as fp32
// [64 columns][128 rows + 1] (the padding keeps both the transposing writes
// and the per-column reads on distinct banks); a thread quantizes one
// 16-row block of one column; codes go through shared memory so each
// column's 64 bytes of codes are stored contiguously.
// ---------------------------------------------------------------------------
constexpr int kColR = 128, kColC = 64, kColThreads = 256;

// SR: stochastic rounding of the codes with the row-wise quantizer's bits,
// taken over x^T: block (c, r / 16) of x^T [C, R] uses the four outputs of
// the generator at counter c * (R / 16) + r / 16 (its flat block index).
template <typename T, bool SR = false>
__global__ void __launch_bounds__(kColThreads) k_nvfp4_quantize_columnwise(
    const T* __restrict__ x, uint32_t R, uint32_t C, const float* __restrict__ g, uint32_t* __restrict__ codes,
    ScaleOut so, uint64_t seed = 0) {
  __shared__ float tile[kColC][kColR + 1];
  __shared__ uint2 qcodes[kColC][kColR / 16];
  const float E = g ? kGlobalEncode / __ldg(g) : 1.0f;
  const uint32_t r0 = blockIdx.x * kColR, c0 = blockIdx.y * kColC;
  // load: a thread takes 8 consecutive columns of a row (one vector load
  // when they are in range and C % 8 == 0); for a fixed element the 32 lanes
  // (8 column groups x 4 rows) write 32 distinct banks of the padded tile
  for (uint32_t i = threadIdx.x; i < (uint32_t)(kColR * kColC / 8); i += blockDim.x) {
    const uint32_t rr = i / (kColC / 8), cg = i % (kColC / 8);
    const uint32_t r = r0 + rr, c = c0 + cg * 8u;
    float v[8];
    if (r < R && c + 8u <= C && (C & 7u) == 0) {
      load8<T>(x + (size_t)r * C + c, v);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = (r < R && c + j < C) ? Elem<T>::to_f(x[(size_t)r * C + c + j]) : 0.0f;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) tile[cg * 8u + j][rr] = v[j];
  }
  __syncthreads();
  // quantize: unit (column cc, row block rb), consecutive lanes on consecutive columns
  for (uint32_t u = threadIdx.x; u < (uint32_t)(kColC * (kColR / 16)); u += blockDim.x) {
    const uint32_t cc = u % kColC, rb = u / kColC;
    float v[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = tile[cc][rb * 16 + j];
    float a = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) a = fmaxf(a, fabsf(v[j]));
    float t = a / kE2M1Max;
    t = t * E;
    const uint32_t s = f32_to_e4m3(t);
    const float fs = e4m3_to_f32(s);
    uint32_t w0 = 0, w1 = 0;
    const uint32_t c = c0 + cc, r = r0 + rb * 16;
    if constexpr (SR) {
      const uint4 r4 = philox4x32_10(make_uint4(c * (R / 16u) + r / 16u, 0u, 0u, 0u), (uint32_t)seed,
                                     (uint32_t)(seed >> 32));
      if (fs != 0.0f) {
        const float k = E / fs;
        const uint32_t rw[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          w0 |= e2m1_sr(v[j] * k, (rw[j >> 2] >> (8 * (j & 3))) & 0xFFu) << (4 * j);
          w1 |= e2m1_sr(v[8 + j] * k, (rw[2 + (j >> 2)] >> (8 * (j & 3))) & 0xFFu) << (4 * j);
        }
      }
    } else if (fs != 0.0f) {
      const float k = E / fs;
      float q0[8], q1[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        q0[j] = v[j] * k;
        q1[j] = v[8 + j] * k;
      }
      w0 = f32x8_to_e2m1x8(q0);
      w1 = f32x8_to_e2m1x8(q1);
    }
    qcodes[cc][rb] = make_uint2(w0, w1);
    if (c < C && r < R) so.store(c * (R / 16u) + r / 16u, s);
  }
  __syncthreads();
  // store: column cc of the tile is row c of x^T, its 16 blocks 128 contiguous bytes
  const uint32_t wpr = R / 8u;  // code words per row of x^T
  for (uint32_t i = threadIdx.x; i < (uint32_t)(kColC * (kColR / 16)); i += blockDim.x) {
    const uint32_t cc = i / (kColR / 16), rb = i % (kColR / 16);
    const uint32_t c = c0 + cc, r = r0 + rb * 16;
    if (c < C && r < R) *reinterpret_cast<uint2*>(codes + (size_t)c * wpr + r / 8u) = qcodes[cc][rb];
  }
  zero_scale_padding(so, C);
}

// ---------------------------------------------------------------------------
// a11: MXFP8 quantize (fp_quantize_rowwise with bits 8 and the e8m0 scale;
// the scale is rounded up, as the mlxcel note on the "[Metal] global scale
// for qmm" page records for CUDA):  per 32-block: v = max|x| / 448;
//   s = ue8m0 rounded up (v);  k = 1 / 2^(s-127);  q_i = e4m3_rne_satfinite(x_i * k)
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kEwThreads) k_mxfp8_quantize(
    const T* __restrict__ x, uint32_t n_half, uint32_t* __restrict__ codes, ScaleOut so,
    uint32_t rows) {
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  for (uint32_t base = warp * 32u * kUnroll; base < n_half; base += nwarps * 32u * kUnroll) {
    float v[kUnroll][8];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t hb = base + u * 32u + lane;
      if (hb < n_half) {
        load8<T>(x + (size_t)hb * 8, v[u]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[u][j] = 0.0f;
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t hb = base + u * 32u + lane;
      float a = 0.0f;
#pragma unroll
      for (int j = 0; j < 8; ++j) a = fmaxf(a, fabsf(v[u][j]));
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
      const float sv = a / kE4M3Max;
      const uint32_t s = f32_to_ue8m0_rp(sv);
      const float k = 1.0f / ue8m0_to_f32(s);
      const uint32_t w0 = f32x4_to_e4m3x4(v[u][0] * k, v[u][1] * k, v[u][2] * k, v[u][3] * k);
      const uint32_t w1 = f32x4_to_e4m3x4(v[u][4] * k, v[u][5] * k, v[u][6] * k, v[u][7] * k);
      if (hb < n_half) {
        reinterpret_cast<uint2*>(codes)[hb] = make_uint2(w0, w1);
        if ((lane & 3u) == 0) so.store(hb >> 2, s);
      }
    }
  }
  zero_scale_padding(so, rows);
}

// ---------------------------------------------------------------------------
// MXFP4 quantize (fp_quantize_rowwise with bits 4 and the e8m0 scale, "mlx
// 0.30.7.2 -> 0.30.7.6" diff, page 7; the scale rounded up as for MXFP8):
// per 32-block: v = max|x| / 6;  s = ue8m0 rounded up (v);
//   k = 1 / 2^(s-127);  q_i = e2m1_rne_satfinite(x_i * k), 8 codes per word
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kEwThreads) k_mxfp4_quantize(
    const T* __restrict__ x, uint32_t n_half, uint32_t* __restrict__ codes, ScaleOut so,
    uint32_t rows) {
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  for (uint32_t base = warp * 32u * kUnroll; base < n_half; base += nwarps * 32u * kUnroll) {
    float v[kUnroll][8];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t hb = base + u * 32u + lane;
      if (hb < n_half) {
        load8<T>(x + (size_t)hb * 8, v[u]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[u][j] = 0.0f;
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t hb = base + u * 32u + lane;
      float a = 0.0f;
#pragma unroll
      for (int j = 0; j < 8; ++j) a = fmaxf(a, fabsf(v[u][j]));
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
      const float sv = a / kE2M1Max;
      const uint32_t s = f32_to_ue8m0_rp(sv);
      const float k = 1.0f / ue8m0_to_f32(s);
      float q[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) q[j] = v[u][j] * k;
      const uint32_t w = f32x8_to_e2m1x8(q);
      if (hb < n_half) {
        codes[hb] = w;
        if ((lane & 3u) == 0) so.store(hb >> 2, s);
      }
    }
  }
  zero_scale_padding(so, rows);
}

// Scale byte of block `block` from a LINEAR or 128x4-tile buffer.
struct ScaleIn {
  const uint8_t* p;
  uint32_t blocks_per_row;
  uint32_t Cp;
  bool swizzled;
  __device__ __forceinline__ uint32_t load(uint32_t block) const {
    if (!swizzled) return __ldg(p + block);
    uint32_t r = block / blocks_per_row, c = block - r * blocks_per_row;
    return __ldg(p + swizzled_offset(r, c, Cp));
  }
};

// ---------------------------------------------------------------------------
// a5: NVFP4 dequantize ("mlx 0.30.7.2 -> 0.30.7.6" diff, page 7,
// fp_dequantize with global scale): w_hat = T(e2m1(q) * (f8(s) * (g / 2688))).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kEwThreads) k_nvfp4_dequantize(
    const uint32_t* __restrict__ codes, ScaleIn si, const float* __restrict__ g,
    uint32_t n_half, T* __restrict__ out) {
  const float d = g ? __ldg(g) / kGlobalEncode : 1.0f;
  const uint32_t tid = blockIdx.x * blockDim.x + threadIdx.x, nthr = gridDim.x * blockDim.x;
  for (uint32_t hb = tid; hb < n_half; hb += nthr) {
    const uint32_t w = __ldg(codes + hb);
    const float sd = e4m3_to_f32(si.load(hb >> 1)) * d;
    float v[8];
    e2m1x8_to_f32(w, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = v[j] * sd;
    store8<T>(out + (size_t)hb * 8, v);
  }
}

// MXFP8 dequantize ("mlx 0.30.7.2 -> 0.30.7.6" diff, page 8, ops.cpp
// fp_dequantize fallback, e8m0 branch): w_hat = T(e4m3(q) * 2^(s-127)).
template <typename T>
__global__ void __launch_bounds__(kEwThreads) k_mxfp8_dequantize(
    const uint32_t* __restrict__ codes, ScaleIn si, uint32_t n_half, T* __restrict__ out) {
  const uint32_t tid = blockIdx.x * blockDim.x + threadIdx.x, nthr = gridDim.x * blockDim.x;
  for (uint32_t hb = tid; hb < n_half; hb += nthr) {
    const uint2 w = __ldg(reinterpret_cast<const uint2*>(codes) + hb);
    const float sc = ue8m0_to_f32(si.load(hb >> 2));
    float a[4], b[4], v[8];
    e4m3x4_to_f32(w.x, a);
    e4m3x4_to_f32(w.y, b);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[j] = a[j] * sc;
      v[4 + j] = b[j] * sc;
    }
    store8<T>(out + (size_t)hb * 8, v);
  }
}

// MXFP4 dequantize (fp_dequantize, e8m0 branch with 4-bit codes):
//   w_hat = T(e2m1(q) * 2^(s-127)).
template <typename T>
__global__ void __launch_bounds__(kEwThreads) k_mxfp4_dequantize(
    const uint32_t* __restrict__ codes, ScaleIn si, uint32_t n_half, T* __restrict__ out) {
  const uint32_t tid = blockIdx.x * blockDim.x + threadIdx.x, nthr = gridDim.x * blockDim.x;
  for (uint32_t hb = tid; hb < n_half; hb += nthr) {
    const uint32_t w = __ldg(codes + hb);
    const float sc = ue8m0_to_f32(si.load(hb >> 2));
    float v[8];
    e2m1x8_to_f32(w, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = v[j] * sc;
    store8<T>(out + (size_t)hb * 8, v);
  }
}

// Standalone LINEAR -> 128x4-tile re-layout of a [rows, cols] scale matrix,
// with zero padding ("mlx 0.30.7" diff, page 71, qqmm_utils.cu swizzle_scales).
// One thread per output byte: every byte of the padded buffer is written.
__global__ void __launch_bounds__(kEwThreads) k_swizzle_scales(
    const uint8_t* __restrict__ lin, uint32_t rows, uint32_t cols, uint32_t Rp, uint32_t Cp,
    uint8_t* __restrict__ swz) {
  const uint32_t tid = blockIdx.x * blockDim.x + threadIdx.x, nthr = gridDim.x * blockDim.x;
  const uint32_t total = Rp * Cp;
  for (uint32_t o = tid; o < total; o += nthr) {
    // invert the tile offset: o = (tile * 512) + (r%32)*16 + ((r%128)/32)*4 + c%4
    const uint32_t tile = o >> 9, in = o & 511u;
    const uint32_t rb = tile / (Cp >> 2), cb = tile - rb * (Cp >> 2);
    const uint32_t r = rb * 128u + ((in >> 2) & 3u) * 32u + (in >> 4);
    const uint32_t c = cb * 4u + (in & 3u);
    swz[o] = (r < rows && c < cols) ? __ldg(lin + (size_t)r * cols + c) : (uint8_t)0;
  }
}

}  // namespace nvfp4
