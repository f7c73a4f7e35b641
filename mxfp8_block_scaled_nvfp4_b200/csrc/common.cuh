// Device helpers shared by the NVFP4 / MXFP8 kernels (sm_100a).
//
// Conversions use the sm_100a cvt instructions directly (round to nearest
// even with saturation to the largest finite value for e2m1 / e4m3, round
// up for ue8m0).  Nothing here uses fast-math: the quantizer's scale
// arithmetic must be IEEE fp32 division and multiplication, in the order of
// the fp_quantize_rowwise kernel ("mlx 0.30.7.2 -> 0.30.7.6" diff, page 7,
// fp_quantize.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace nvfp4 {

// 448 (largest e4m3) times 6 (largest e2m1): the global encode constant of
// NVFP4's two-level scale (fp_quantize.cu: F8E4M3_MAX * F4E2M1_MAX).
constexpr float kE4M3Max = 448.0f;
constexpr float kE2M1Max = 6.0f;
constexpr float kGlobalEncode = kE4M3Max * kE2M1Max;

// Device error word, set by kernels that detect a bad input (an expert index
// out of range) or give up a bounded wait; read and cleared by the host.
enum DeviceError : unsigned int {
  kDevErrNone = 0,
  kDevErrIndex = 1,
  kDevErrTimeout = 2,
};

// The library is one translation unit, so this is its only definition.
__device__ unsigned int g_device_error = 0;

// ---------------------------------------------------------------------------
// element types
// ---------------------------------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float v) { return v; }
  static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Elem<__half> {
  static __device__ __forceinline__ float to_f(__half v) { return __half2float(v); }
  static __device__ __forceinline__ __half from_f(float v) { return __float2half_rn(v); }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

// 8 consecutive elements held in one 16-byte word (2-byte types) or two
// (fp32), as fp32.
template <typename T>
__device__ __forceinline__ void unpack8(uint4 a, uint4 b, float (&v)[8]);

template <>
__device__ __forceinline__ void unpack8<float>(uint4 a, uint4 b, float (&v)[8]) {
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(w[i]);
}

template <>
__device__ __forceinline__ void unpack8<__nv_bfloat16>(uint4 u, uint4, float (&v)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <>
__device__ __forceinline__ void unpack8<__half>(uint4 u, uint4, float (&v)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
        : "=f"(v[2 * i]), "=f"(v[2 * i + 1])
        : "r"(w[i]));
  }
}

// Load 8 consecutive elements (16 B for 2-byte types, 32 B for fp32) of
// global memory as fp32 (read-only path).
template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&v)[8]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
  unpack8<T>(__ldg(q), sizeof(T) == 4 ? __ldg(q + 1) : make_uint4(0, 0, 0, 0), v);
}

// The same from shared memory (generic loads).
template <typename T>
__device__ __forceinline__ void load8_shared(const T* p, float (&v)[8]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
  unpack8<T>(q[0], sizeof(T) == 4 ? q[1] : make_uint4(0, 0, 0, 0), v);
}

// Store 8 fp32 values rounded to T (RNE).
template <typename T>
__device__ __forceinline__ void store8(T* p, const float (&v)[8]);

template <>
__device__ __forceinline__ void store8<float>(float* p, const float (&v)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

// Two fp32 values rounded (RNE) to a packed bf16x2 / f16x2 word, `lo` in
// the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

template <>
__device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16* p, const float (&v)[8]) {
  *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                            pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}

template <>
__device__ __forceinline__ void store8<__half>(__half* p, const float (&v)[8]) {
  *reinterpret_cast<uint4*>(p) = make_uint4(pack_f16x2(v[0], v[1]), pack_f16x2(v[2], v[3]),
                                            pack_f16x2(v[4], v[5]), pack_f16x2(v[6], v[7]));
}

// ---------------------------------------------------------------------------
// format conversions (sm_100a cvt)
// ---------------------------------------------------------------------------

// e4m3, round to nearest even, saturate to +-448.  Returns the byte.
__device__ __forceinline__ uint32_t f32_to_e4m3(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return r & 0xFFu;
}

// ue8m0, rounded up (toward +infinity), saturated.  Returns the byte.
__device__ __forceinline__ uint32_t f32_to_ue8m0_rp(float v) {
  uint16_t r;
  asm("cvt.rp.satfinite.ue8m0x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return r & 0xFFu;
}

// Value of an e4m3 byte (exact: e4m3 is a subset of fp16).
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
  float f;
  asm("{\n\t.reg .b16 in, l, h;\n\t.reg .b32 p;\n\t"
      "cvt.u16.u32 in, %1;\n\t"
      "cvt.rn.f16x2.e4m3x2 p, in;\n\t"
      "mov.b32 {l, h}, p;\n\t"
      "cvt.f32.f16 %0, l;\n\t}"
      : "=f"(f)
      : "r"(b & 0xFFu));
  return f;
}

// Value of a ue8m0 byte: 2^(b-127) (b = 0 gives the fp32 subnormal 2^-127).
__device__ __forceinline__ float ue8m0_to_f32(uint32_t b) {
  return b == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(b << 23);
}

// Eight fp32 values to eight e2m1 codes (RNE, satfinite), element i in bits
// 4i..4i+3 of the result.
__device__ __forceinline__ uint32_t f32x8_to_e2m1x8(const float (&v)[8]) {
  uint32_t out;
  asm("{\n\t"
      ".reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t"
      "}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return out;
}

// e2m1 codes of v[i] * k (each product rounded to fp32, as v[i] * k is;
// computed two at a time by the packed fp32x2 multiply), element i in bits
// 4i..4i+3.
__device__ __forceinline__ uint32_t scaled_e2m1x8(const float (&v)[8], float k) {
  uint32_t out;
  asm("{\n\t"
      ".reg .b64 kk, p0, p1, p2, p3;\n\t"
      ".reg .f32 q0, q1, q2, q3, q4, q5, q6, q7;\n\t"
      ".reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b64 kk, {%9, %9};\n\t"
      "mov.b64 p0, {%1, %2};\n\t"
      "mov.b64 p1, {%3, %4};\n\t"
      "mov.b64 p2, {%5, %6};\n\t"
      "mov.b64 p3, {%7, %8};\n\t"
      "mul.rn.f32x2 p0, p0, kk;\n\t"
      "mul.rn.f32x2 p1, p1, kk;\n\t"
      "mul.rn.f32x2 p2, p2, kk;\n\t"
      "mul.rn.f32x2 p3, p3, kk;\n\t"
      "mov.b64 {q0, q1}, p0;\n\t"
      "mov.b64 {q2, q3}, p1;\n\t"
      "mov.b64 {q4, q5}, p2;\n\t"
      "mov.b64 {q6, q7}, p3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, q1, q0;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, q3, q2;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, q5, q4;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, q7, q6;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t"
      "}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(k));
  return out;
}

// n / d for a fixed divisor d >= 1 and n < 2^31 with one multiply-high
// (Granlund and Montgomery, "Division by invariant integers using
// multiplication", PLDI 1994): with l = ceil(log2 d) and
// m = floor(2^32 (2^l - d) / d) + 1, n / d = (umulhi(n, m) + n) >> l.
struct FastDiv {
  uint32_t d, m, l;
  __host__ __device__ void init(uint32_t dd) {
    d = dd;
    l = 0;
    while ((1ull << l) < (unsigned long long)d) ++l;
    m = (uint32_t)((((1ull << 32) * ((1ull << l) - d)) / d) + 1ull);
  }
  __device__ __forceinline__ uint32_t div(uint32_t n) const { return (__umulhi(n, m) + n) >> l; }
};

// Four fp32 values to four e4m3 bytes (RNE, satfinite), element i in byte i.
__device__ __forceinline__ uint32_t f32x4_to_e4m3x4(float a, float b, float c, float d) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return (uint32_t)lo | ((uint32_t)hi << 16);
}

// Two e2m1 codes in the low byte of `b` to fp32 values (exact).  The byte
// reaches the .b8 operand of the conversion through cvt.u8.u32.
__device__ __forceinline__ void e2m1x2_to_f32(uint32_t b, float& lo, float& hi) {
  asm("{\n\t.reg .b8 q;\n\t.reg .b16 l, h;\n\t.reg .b32 p;\n\t"
      "cvt.u8.u32 q, %2;\n\t"
      "cvt.rn.f16x2.e2m1x2 p, q;\n\t"
      "mov.b32 {l, h}, p;\n\t"
      "cvt.f32.f16 %0, l;\n\t"
      "cvt.f32.f16 %1, h;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(b));
}

// Eight e2m1 codes (element i in bits 4i..4i+3) to their values.
__device__ __forceinline__ void e2m1x8_to_f32(uint32_t codes, float (&v)[8]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) e2m1x2_to_f32((codes >> (8 * i)) & 0xFFu, v[2 * i], v[2 * i + 1]);
}

// Value of a 4-bit e2m1 code by arithmetic: the magnitude bits placed at
// fp32 bits 22-24 read as 2^-126 times the e2m1 value (code 1 lands on the
// subnormal 2^-127 = 0.5 * 2^-126), the sign at bit 31; one exact multiply.
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  return __uint_as_float(((c & 8u) << 28) | ((c & 7u) << 22)) * 0x1p126f;
}

// Four e4m3 bytes (element i in byte i) to their values.
__device__ __forceinline__ void e4m3x4_to_f32(uint32_t codes, float (&v)[4]) {
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    asm("{\n\t.reg .b16 in, l, h;\n\t.reg .b32 p;\n\t"
        "cvt.u16.u32 in, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 p, in;\n\t"
        "mov.b32 {l, h}, p;\n\t"
        "cvt.f32.f16 %0, l;\n\t"
        "cvt.f32.f16 %1, h;\n\t}"
        : "=f"(v[2 * i]), "=f"(v[2 * i + 1])
        : "r"((codes >> (16 * i)) & 0xFFFFu));
  }
}

// ---------------------------------------------------------------------------
// 128x4 scale tiles of the block-scaled MMA ("mlx 0.30.7" diff, page 71,
// qqmm_utils.cu: reshape(rb, 4, 32, cb, 4).transpose(0, 3, 2, 1, 4)):
// byte offset of scale (r, c) in a [ceil128(rows), Cp] buffer, Cp % 4 == 0.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t swizzled_offset(uint32_t r, uint32_t c, uint32_t Cp) {
  return ((r >> 7) * (Cp >> 2) + (c >> 2)) * 512u + (r & 31u) * 16u + ((r >> 5) & 3u) * 4u + (c & 3u);
}

}  // namespace nvfp4
