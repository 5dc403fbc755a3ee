// Squared norms as tensor-core operands.
//
// FlashAssign ranks centroids by ||x - c||^2 = ||x||^2 - 2 x.c + ||c||^2.
// Adding the norms in the epilogue would make every epilogue thread read
// ||c||^2 for each of its columns (shared-memory traffic that competes with the
// tensor core's own operand reads) and spend an FMA per value.  Instead one
// extra MMA step of K = 16 per chunk adds them to the accumulator:
//
//   acc[i][k] = x_i . c_k + sum_e A_ext[i][e] * B_ext[k][e]
//
// Each norm / 2 is split into a few 16-bit "digits" whose scaled sum gives it
// back to fp32 precision; the products are exact in the tensor core and are
// accumulated in fp32.  Extension row layout (16 elements, 32 bytes):
//
//   pos    B side (per centroid, cnx)      A side, packed-key mode     A side, exact mode
//   0..4   digits t of ||c||^2 / 2         -S_e                        -S_e
//   5..9   -S_e                            digits u of ||x||^2 w / 2   0
//   10     2^-14 (bias)                    -1                          0
//   11..15 0                               0                           0
//
// with w = 1 + 2^-10.  Packed-key mode (resident point tile) therefore gets
//   acc = -(||x - c||^2 + 2^-10 ||x||^2) / 2 - 2^-14,
// which is strictly negative, so the float bits of acc order like its
// magnitude and a column index can be packed into the low mantissa bits.
// Exact mode gets acc = x . c - ||c||^2 / 2 (the argmax is the nearest centroid).
//
// fp16: five digits with scales S = 2^15, 2^8, 2^1, 2^-6, 2^-13 (all normal
// fp16 numbers) cover values up to 65504 * 2^15 (about 2^31) with better than
// fp32 precision (each digit carries 11 bits and the scales are 7 bits apart).
// bf16: three digits with S = 1 (8 significand bits each, 24 in total; bf16
// has the fp32 range, so nothing clamps).
// Centroid rows past K get a sentinel row whose acc is about -2^31 (fp16) or
// -2^64 (bf16), so padded columns never win.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace fk {

constexpr int kExt = 16;        // extension K (one MMA step)
constexpr int kExtDigits = 5;   // digits per norm (fp16; bf16 uses 3 of them)
constexpr int kExtXnOff = 5;    // first position of the per-point digits
constexpr int kExtBiasPos = 10; // position of the constant bias

__device__ __forceinline__ float ext_scale_f16(int e) {
  return e == 0 ? 32768.f : e == 1 ? 256.f : e == 2 ? 2.f : e == 3 ? 0.015625f : 0.0001220703125f;
}

// Digits of v >= 0 (fp16).  Returns true when v is beyond the representable
// range (the top digit is clamped).
__device__ __forceinline__ bool ext_digits(float v, __half (&t)[kExtDigits]) {
  bool clamped = false;
  float r = v;
#pragma unroll
  for (int e = 0; e < kExtDigits; ++e) {
    const float s = ext_scale_f16(e);
    float q = r * (1.f / s);  // exact: s is a power of two
    if (q > 65504.f) { q = 65504.f; clamped = true; }
    if (q < -65504.f) { q = -65504.f; clamped = true; }
    const __half h = __float2half_rn(q);
    t[e] = h;
    r = fmaf(-__half2float(h), s, r);  // exact residual
  }
  return clamped;
}

// Digits of v >= 0 (bf16): v = t0 + t1 + t2 to 24 bits; t3 = t4 = 0.
__device__ __forceinline__ bool ext_digits(float v, __nv_bfloat16 (&t)[kExtDigits]) {
  float r = v;
#pragma unroll
  for (int e = 0; e < 3; ++e) {
    const __nv_bfloat16 h = __float2bfloat16_rn(r);
    t[e] = h;
    r = r - __bfloat162float(h);
  }
  t[3] = __float2bfloat16_rn(0.f);
  t[4] = __float2bfloat16_rn(0.f);
  return false;
}

template <typename T> __device__ __forceinline__ T ext_val(float v);
template <> __device__ __forceinline__ __half ext_val<__half>(float v) { return __float2half_rn(v); }
template <> __device__ __forceinline__ __nv_bfloat16 ext_val<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

template <typename T> __device__ __forceinline__ T ext_neg_scale(int e);
template <> __device__ __forceinline__ __half ext_neg_scale<__half>(int e) {
  return __float2half_rn(-ext_scale_f16(e));
}
template <> __device__ __forceinline__ __nv_bfloat16 ext_neg_scale<__nv_bfloat16>(int e) {
  return __float2bfloat16_rn(e < 3 ? -1.f : 0.f);
}

// Digit e of the sentinel row of a padded centroid: every fp16 digit at its
// maximum (acc about -2^31), or 2^64 in the first bf16 digit.
template <typename T> __device__ __forceinline__ T ext_sentinel(int e);
template <> __device__ __forceinline__ __half ext_sentinel<__half>(int) { return __float2half_rn(65504.f); }
template <> __device__ __forceinline__ __nv_bfloat16 ext_sentinel<__nv_bfloat16>(int e) {
  return __float2bfloat16_rn(e == 0 ? 18446744073709551616.f : 0.f);
}

// The B-side row of one centroid from ||c||^2 (real) or the sentinel row.
template <typename T>
__device__ __forceinline__ bool ext_centroid_row(float cn, bool real, T (&row)[kExt]) {
  bool clamped = false;
  T t[kExtDigits];
  if (real) {
    clamped = ext_digits(0.5f * cn, t);
  } else {
#pragma unroll
    for (int e = 0; e < kExtDigits; ++e) t[e] = ext_sentinel<T>(e);
  }
#pragma unroll
  for (int e = 0; e < kExtDigits; ++e) {
    row[e] = t[e];
    row[kExtXnOff + e] = ext_neg_scale<T>(e);
  }
  row[kExtBiasPos] = ext_val<T>(0.00006103515625f);  // 2^-14
#pragma unroll
  for (int e = kExtBiasPos + 1; e < kExt; ++e) row[e] = ext_val<T>(0.f);
  return clamped;
}

// The A-side row of one point: packed-key mode from ||x||^2, or the exact-mode
// constant row (xn2 ignored).
template <typename T, bool PACKED>
__device__ __forceinline__ bool ext_point_row(float xn2, T (&row)[kExt]) {
  bool clamped = false;
  T u[kExtDigits];
  if (PACKED) {
    clamped = ext_digits(fmaf(xn2, 0.5f * 0.0009765625f, 0.5f * xn2), u);
  }
#pragma unroll
  for (int e = 0; e < kExtDigits; ++e) {
    row[e] = ext_neg_scale<T>(e);
    row[kExtXnOff + e] = PACKED ? u[e] : ext_val<T>(0.f);
  }
  row[kExtBiasPos] = ext_val<T>(PACKED ? -1.f : 0.f);
#pragma unroll
  for (int e = kExtBiasPos + 1; e < kExt; ++e) row[e] = ext_val<T>(0.f);
  return clamped;
}

// tf32 (fp32 points on the tensor cores, kind::tf32, exact mode only): a row
// is 8 fp32 values (32 bytes, one K = 8 step).  ||c||^2 / 2 is split into
// three tf32 digits (the value truncated to 10 fraction bits, then the exact
// remainder truncated the same way, then the rest, which has at most 2
// significant bits left), so the digits sum back to the fp32 value exactly.
//   B side: [t0, t1, t2, 0, 0, 0, 0, 0]   A side: [-1, -1, -1, 0, 0, 0, 0, 0]
// giving acc = x.c - ||c||^2 / 2.  A padded centroid gets t0 = 2^100.
constexpr int kExtF32 = 8;

__device__ __forceinline__ float tf32_trunc(float v) {
  return __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
}

__device__ __forceinline__ void ext_centroid_row_f32(float cn, bool real, float (&row)[kExtF32]) {
#pragma unroll
  for (int e = 0; e < kExtF32; ++e) row[e] = 0.f;
  if (!real) {
    row[0] = 1267650600228229401496703205376.f;  // 2^100
    return;
  }
  float r = 0.5f * cn;
#pragma unroll
  for (int e = 0; e < 3; ++e) {
    const float t = e < 2 ? tf32_trunc(r) : r;
    row[e] = t;
    r -= t;  // exact: t holds leading bits of r
  }
}

__device__ __forceinline__ void ext_point_row_f32(float (&row)[kExtF32]) {
#pragma unroll
  for (int e = 0; e < kExtF32; ++e) row[e] = e < 3 ? -1.f : 0.f;
}

}  // namespace fk
