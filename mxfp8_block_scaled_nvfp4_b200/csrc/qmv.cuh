// qmv: the small-M route of qqmm with a pre-quantized NVFP4 weight
// ("mlx 0.30.7.2 -> 0.30.7.6" diff, page 7, qqmm.cpp, QQMatmul::eval_gpu:
// when w is quantized and x has one row, x is quantize-dequantized with its
// global scale and fp_qmv multiplies it with w).
//
//   x_hat[m, k] = T(e2m1(qx) * (f8(sx) * g_x / 2688))     (per 16-block of x)
//   y[m, n]     = T( sum_b sd[n, b] * sum_{k in b} x_hat[m, k] * e2m1(qw[n, k]) )
//   sd[n, b]    = f8(sw[n, b]) * (g_w / 2688)              (fp32)
//
// The weight's global scale multiplies each block scale (osaurus-ai/mlx
// pull 31, "The fix": per block, not on the sum); the weight itself is not
// rounded to T on this path, so the block scale can be applied once per
// block sum (exact in real arithmetic).  Accumulation is fp32.
//
// Kernel shape.  Every CTA first builds x_hat for all M rows in shared
// memory as fp32 (M * K * 4 bytes).  x_hat is stored in 32-element chunks
// whose eight 16-byte segments are XOR-swizzled by the chunk index, so the
// 8 lanes of a 128-bit shared load phase hit distinct banks.  Each warp then
// owns weight rows n = warp, warp + nwarps, ...; lane l reads 128-bit code
// chunks l, l+32, l+64, l+96 of a row (one coalesced 512-byte load per warp
// and chunk step) and their two scale bytes, with the next row's loads
// issued before the current row is computed (register double buffering),
// so 128 bytes per lane are in flight.  The row sum is a warp shuffle
// reduction.  W is streamed once from HBM: 0.5625 bytes per weight.
#pragma once

#include "common.cuh"

namespace nvfp4 {

constexpr int kQmvThreads = 512;
constexpr int kQmvMaxM = 8;
constexpr int kQmvCH = 4;  // 128-bit chunks per lane per unit

// fp32 index of element k of row m in the swizzled x_hat layout.
__device__ __forceinline__ uint32_t xs_index(uint32_t m, uint32_t K, uint32_t k) {
  const uint32_t c = k >> 5, seg = (k >> 2) & 7u;
  return m * K + (c << 5) + ((seg ^ (c & 7u)) << 2) + (k & 3u);
}

// x_hat = quantize-dequantize(x, g_x) ("fp_quantize_dequantize") for all M
// rows into shared memory (fp32, swizzled chunks).
template <typename T>
__device__ __forceinline__ void qmv_prologue(const T* __restrict__ x, const float* __restrict__ g_x, uint32_t M,
                                             uint32_t K, float4* xs4, uint32_t thread, uint32_t nthreads) {
  const uint32_t lane = threadIdx.x & 31u;
  const float E = g_x ? kGlobalEncode / __ldg(g_x) : 1.0f;
  const float d = g_x ? __ldg(g_x) / kGlobalEncode : 1.0f;
  const uint32_t n_half = M * K / 8u;
  for (uint32_t base = (thread & ~31u); base < n_half; base += nthreads) {
    const uint32_t hb = base + lane;
    float v[8];
    if (hb < n_half) {
      load8<T>(x + (size_t)hb * 8, v);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = 0.0f;
    }
    float a = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) a = fmaxf(a, fabsf(v[j]));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
    float t = a / kE2M1Max;
    t = t * E;
    const uint32_t s = f32_to_e4m3(t);
    const float fs = e4m3_to_f32(s);
    float dq[8];
    const float sd = fs * d;
    if (fs != 0.0f) {
      const float k = E / fs;
      float q[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) q[j] = v[j] * k;
      const uint32_t w = f32x8_to_e2m1x8(q);
#pragma unroll
      for (int j = 0; j < 8; ++j) dq[j] = Elem<T>::to_f(Elem<T>::from_f(e2m1_value(w >> (4 * j)) * sd));
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) dq[j] = 0.0f;
    }
    if (hb < n_half) {
      const uint32_t m = (hb * 8u) / K, k0 = hb * 8u - m * K;
      const uint32_t i0 = xs_index(m, K, k0), i1 = xs_index(m, K, k0 + 4);
      xs4[i0 >> 2] = make_float4(dq[0], dq[1], dq[2], dq[3]);
      xs4[i1 >> 2] = make_float4(dq[4], dq[5], dq[6], dq[7]);
    }
  }
}

// y rows n = first, first + step, ... < end (one warp per row) from x_hat in
// shared memory: coalesced 128-bit code loads with register double buffering.
template <typename T, int MM>
__device__ __forceinline__ void qmv_simt_rows(const float4* xs4, const uint32_t* __restrict__ wc,
                                              const uint8_t* __restrict__ ws, float dw, uint32_t M, uint32_t N,
                                              uint32_t K, T* __restrict__ y, uint32_t first, uint32_t step,
                                              uint32_t end) {
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t chunks = K >> 5;  // 32 codes (16 bytes) per chunk
  const uint32_t groups = (chunks + 32u * kQmvCH - 1) / (32u * kQmvCH);
  const uint4* wc4 = reinterpret_cast<const uint4*>(wc);
  uint32_t un = first, ug = 0;
  uint4 qb[kQmvCH];
  uint32_t sb[kQmvCH];
  auto load_unit = [&](uint32_t n, uint32_t g) {
#pragma unroll
    for (int i = 0; i < kQmvCH; ++i) {
      const uint32_t c = g * 32u * kQmvCH + (uint32_t)i * 32u + lane;
      if (n < end && c < chunks) {
        qb[i] = __ldg(wc4 + (size_t)n * chunks + c);
        sb[i] = __ldg(reinterpret_cast<const unsigned short*>(ws + (size_t)n * (chunks * 2u) + 2u * c));
      } else {
        qb[i] = make_uint4(0, 0, 0, 0);
        sb[i] = 0;
      }
    }
  };
  load_unit(un, ug);
  float acc[MM];
#pragma unroll
  for (int m = 0; m < MM; ++m) acc[m] = 0.0f;
  while (un < end) {
    uint4 q[kQmvCH];
    uint32_t s[kQmvCH];
#pragma unroll
    for (int i = 0; i < kQmvCH; ++i) {
      q[i] = qb[i];
      s[i] = sb[i];
    }
    const uint32_t cn = un, cg = ug;
    if (++ug == groups) {
      ug = 0;
      un += step;
    }
    load_unit(un, ug);  // next unit's loads in flight while this one computes
#pragma unroll
    for (int i = 0; i < kQmvCH; ++i) {
      const uint32_t c = cg * 32u * kQmvCH + (uint32_t)i * 32u + lane;
      if (c < chunks) {
        const uint32_t wv[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
#pragma unroll
        for (int b = 0; b < 2; ++b) {  // two 16-code blocks per chunk
          const float sd = e4m3_to_f32((s[i] >> (8 * b)) & 0xFFu) * dw;
          float bs[MM];
#pragma unroll
          for (int m = 0; m < MM; ++m) bs[m] = 0.0f;
#pragma unroll
          for (int seg = 0; seg < 4; ++seg) {  // 4-element segments of the block
            const uint32_t word = wv[2 * b + (seg >> 1)] >> (16 * (seg & 1));
            float v0, v1, v2, v3;
            e2m1x2_to_f32(word & 0xFFu, v0, v1);
            e2m1x2_to_f32((word >> 8) & 0xFFu, v2, v3);
            const uint32_t sg = (uint32_t)(4 * b + seg);
            const uint32_t off = (c << 5) + ((sg ^ (c & 7u)) << 2);
#pragma unroll
            for (int m = 0; m < MM; ++m) {
              if ((uint32_t)m < M) {
                const float4 xv = xs4[(m * K + off) >> 2];
                bs[m] = fmaf(xv.x, v0, bs[m]);
                bs[m] = fmaf(xv.y, v1, bs[m]);
                bs[m] = fmaf(xv.z, v2, bs[m]);
                bs[m] = fmaf(xv.w, v3, bs[m]);
              }
            }
          }
#pragma unroll
          for (int m = 0; m < MM; ++m) acc[m] = fmaf(bs[m], sd, acc[m]);
        }
      }
    }
    if (cg + 1 == groups) {  // row finished: reduce across the warp and store
#pragma unroll
      for (int m = 0; m < MM; ++m) {
        if ((uint32_t)m < M) {
          float a = acc[m];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
          if (lane == 0) y[(size_t)m * N + cn] = Elem<T>::from_f(a);
        }
        acc[m] = 0.0f;
      }
    }
  }
}

template <typename T, int MM>
__global__ void __launch_bounds__(kQmvThreads) k_qmv(
    const T* __restrict__ x, const float* __restrict__ g_x, const uint32_t* __restrict__ wc,
    const uint8_t* __restrict__ ws, const float* __restrict__ g_w, int M_, int N, int K,
    T* __restrict__ y) {
  extern __shared__ float4 xs4[];
  qmv_prologue<T>(x, g_x, (uint32_t)M_, (uint32_t)K, xs4, threadIdx.x, blockDim.x);
  __syncthreads();
  const float dw = g_w ? __ldg(g_w) / kGlobalEncode : 1.0f;
  const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  qmv_simt_rows<T, MM>(xs4, wc, ws, dw, (uint32_t)M_, (uint32_t)N, (uint32_t)K, y, warp, nwarps, (uint32_t)N);
}

}  // namespace nvfp4

namespace nvfp4 {

// ---------------------------------------------------------------------------
// qmv in the MX modes: the same M = 1 route ("mlx 0.30.7.2 -> 0.30.7.6"
// diff, page 7, qqmm.cpp, QQMatmul::eval_gpu: fp_quantize_dequantize of x
// with the mode's group size and bits, then fp_qmv), with 32-element blocks
// and e8m0 scales rounded up, no global scales:
//   MODE 1 (MXFP8): codes e4m3 (4 per uint32), x_hat[k] = T(e4m3(qx) * 2^(sx-127))
//   MODE 2 (MXFP4): codes e2m1 (8 per uint32), x_hat[k] = T(e2m1(qx) * 2^(sx-127))
//   y[m, n] = T( sum_b 2^(sw[n,b]-127) * sum_{k in b} x_hat[m, k] * code(q[n, k]) ),
// fp32 accumulation (the per-block power of two is exact in fp32).
// Same kernel shape as k_qmv: x_hat for all M rows in shared memory (fp32,
// swizzled 32-element chunks), a warp per weight row, 128-bit coalesced
// code loads with the next unit's loads in flight.
// ---------------------------------------------------------------------------
template <typename T, int MODE>
__device__ __forceinline__ void qmv_mx_prologue(const T* __restrict__ x, uint32_t M, uint32_t K, float4* xs4) {
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t n_half = M * K / 8u;  // 4 half-blocks per 32-block, 8 per warp step
  for (uint32_t base = (threadIdx.x & ~31u); base < n_half; base += blockDim.x) {
    const uint32_t hb = base + lane;
    float v[8];
    if (hb < n_half) {
      load8<T>(x + (size_t)hb * 8, v);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = 0.0f;
    }
    float a = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) a = fmaxf(a, fabsf(v[j]));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
    const uint32_t s = f32_to_ue8m0_rp(a / (MODE == 1 ? kE4M3Max : kE2M1Max));
    const float sc = ue8m0_to_f32(s);
    const float k = 1.0f / sc;
    float dq[8];
    if constexpr (MODE == 1) {
      float c0[4], c1[4];
      e4m3x4_to_f32(f32x4_to_e4m3x4(v[0] * k, v[1] * k, v[2] * k, v[3] * k), c0);
      e4m3x4_to_f32(f32x4_to_e4m3x4(v[4] * k, v[5] * k, v[6] * k, v[7] * k), c1);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        dq[j] = Elem<T>::to_f(Elem<T>::from_f(c0[j] * sc));
        dq[4 + j] = Elem<T>::to_f(Elem<T>::from_f(c1[j] * sc));
      }
    } else {
      float q[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) q[j] = v[j] * k;
      const uint32_t w = f32x8_to_e2m1x8(q);
#pragma unroll
      for (int j = 0; j < 8; ++j) dq[j] = Elem<T>::to_f(Elem<T>::from_f(e2m1_value(w >> (4 * j)) * sc));
    }
    if (hb < n_half) {
      const uint32_t m = (hb * 8u) / K, k0 = hb * 8u - m * K;
      const uint32_t i0 = xs_index(m, K, k0), i1 = xs_index(m, K, k0 + 4);
      xs4[i0 >> 2] = make_float4(dq[0], dq[1], dq[2], dq[3]);
      xs4[i1 >> 2] = make_float4(dq[4], dq[5], dq[6], dq[7]);
    }
  }
}

// Weight row n's chunk c of 128 bits: 32 e2m1 codes (MXFP4, one 32-block)
// or 16 e4m3 codes (MXFP8, half a block) starting at element kc; values
// into v (the codes' values, unscaled).
template <int MODE>
__device__ __forceinline__ void mx_chunk_values(uint4 q, float (&v)[32]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  if constexpr (MODE == 2) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float t[8];
      e2m1x8_to_f32(w[i], t);
#pragma unroll
      for (int j = 0; j < 8; ++j) v[8 * i + j] = t[j];
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float t[4];
      e4m3x4_to_f32(w[i], t);
#pragma unroll
      for (int j = 0; j < 4; ++j) v[4 * i + j] = t[j];
    }
  }
}

template <typename T, int MODE, int MM>
__global__ void __launch_bounds__(kQmvThreads) k_qmv_mx(const T* __restrict__ x, const uint32_t* __restrict__ wc,
                                                      const uint8_t* __restrict__ ws, int M_, int N, int K,
                                                      T* __restrict__ y) {
  extern __shared__ float4 xs4[];
  const uint32_t M = (uint32_t)M_;
  qmv_mx_prologue<T, MODE>(x, M, (uint32_t)K, xs4);
  __syncthreads();
  constexpr uint32_t kPerChunk = MODE == 2 ? 32u : 16u;  // codes per 128-bit chunk
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t chunks = (uint32_t)K / kPerChunk;
  const uint32_t groups = (chunks + 32u * kQmvCH - 1) / (32u * kQmvCH);
  const uint32_t nb = (uint32_t)K / 32u;  // scale bytes per row
  const uint4* wc4 = reinterpret_cast<const uint4*>(wc);
  const uint32_t first = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t step = (gridDim.x * blockDim.x) >> 5;
  uint32_t un = first, ug = 0;
  uint4 qb[kQmvCH];
  uint32_t sb[kQmvCH];
  auto load_unit = [&](uint32_t n, uint32_t g) {
#pragma unroll
    for (int i = 0; i < kQmvCH; ++i) {
      const uint32_t c = g * 32u * kQmvCH + (uint32_t)i * 32u + lane;
      if (n < (uint32_t)N && c < chunks) {
        qb[i] = __ldg(wc4 + (size_t)n * chunks + c);
        sb[i] = __ldg(ws + (size_t)n * nb + (c * kPerChunk) / 32u);
      } else {
        qb[i] = make_uint4(0, 0, 0, 0);
        sb[i] = 127;
      }
    }
  };
  load_unit(un, ug);
  float acc[MM];
#pragma unroll
  for (int m = 0; m < MM; ++m) acc[m] = 0.0f;
  while (un < (uint32_t)N) {
    uint4 q[kQmvCH];
    uint32_t s[kQmvCH];
#pragma unroll
    for (int i = 0; i < kQmvCH; ++i) {
      q[i] = qb[i];
      s[i] = sb[i];
    }
    const uint32_t cn = un, cg = ug;
    if (++ug == groups) {
      ug = 0;
      un += step;
    }
    load_unit(un, ug);  // next unit's loads in flight while this one computes
#pragma unroll
    for (int i = 0; i < kQmvCH; ++i) {
      const uint32_t c = cg * 32u * kQmvCH + (uint32_t)i * 32u + lane;
      if (c < chunks) {
        float v[32];
        mx_chunk_values<MODE>(q[i], v);
        const float sw = ue8m0_to_f32(s[i]);
#pragma unroll
        for (int m = 0; m < MM; ++m) {
          if ((uint32_t)m < M) {
            float bs = 0.0f;
#pragma unroll
            for (int j = 0; j < (int)kPerChunk; j += 4) {
              const uint32_t k = c * kPerChunk + (uint32_t)j;
              const float4 xv = xs4[xs_index(m, (uint32_t)K, k) >> 2];
              bs = fmaf(xv.x, v[j], bs);
              bs = fmaf(xv.y, v[j + 1], bs);
              bs = fmaf(xv.z, v[j + 2], bs);
              bs = fmaf(xv.w, v[j + 3], bs);
            }
            acc[m] = fmaf(bs, sw, acc[m]);
          }
        }
      }
    }
    if (cg + 1 == groups) {  // row finished: reduce across the warp and store
#pragma unroll
      for (int m = 0; m < MM; ++m) {
        if ((uint32_t)m < M) {
          float a = acc[m];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
          if (lane == 0) y[(size_t)m * N + cn] = Elem<T>::from_f(a);
        }
        acc[m] = 0.0f;
      }
    }
  }
}

}  // namespace nvfp4
