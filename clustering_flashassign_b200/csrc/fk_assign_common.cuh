// Device helpers of the FlashAssign kernels: the packed-key and exact running
// argmax over TMEM loads, the point-norm sums of a shared tile, the
// 32-byte-swizzled norm-row stores, and the exact fp64 re-rank of points far
// from every centroid.
#pragma once

#include <cuda.h>

#include "fk_norms.cuh"
#include "fk_sm100.cuh"

namespace fk {

constexpr uint32_t kKeyMask = 0xFFFFFF00u;  // packed keys: column in the low byte

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ float key_hi(float key) {
  return __uint_as_float(__float_as_uint(key) & kKeyMask);
}

// A point whose packed-key winner says ||x - c||^2 > 16 ||x||^2: there the
// 2^-15 merge of the packed keys could exceed the near-tie band 1e-3 ||x||^2,
// so the point is re-ranked exactly.  -key = (||x - c||^2 + 2^-10 ||x||^2) / 2
// + 2^-14 (to 2^-15 relative), so the test is -key > 8 ||x||^2; it always
// holds for x = 0.
constexpr float kFarRatioHalf = 8.f;

// The exact-value paths (split-d) rank by v = x.c - ||c||^2 / 2 =
// (||x||^2 - ||x - c||^2) / 2 in fp32.  Far from the origin compared with
// ||x||, the fp32 rounding of v is set by ||c||^2 and can exceed the near-tie
// band: a row with ||x - c||^2 > 64 ||x||^2, i.e. -2 v > 63 ||x||^2, is
// re-ranked exactly.  Only rows with v < 0 (nearest distance above ||x||^2)
// can qualify, so ||x||^2 is read (or computed) for those alone.  Below the
// threshold ||c|| <= 9 ||x||, and the worst-case fp32 error of v (about
// (d / 16) u ||x|| ||c|| for the MMA's accumulation) stays inside the band for
// d up to a few thousand; typical errors grow as sqrt(d).
constexpr float kFarRatioExactM1 = 63.f;

__device__ __forceinline__ double widen_lo(uint32_t v, __half) {
  return (double)__half2float(__ushort_as_half((unsigned short)(v & 0xFFFFu)));
}
__device__ __forceinline__ double widen_hi(uint32_t v, __half) {
  return (double)__half2float(__ushort_as_half((unsigned short)(v >> 16)));
}
__device__ __forceinline__ double widen_lo(uint32_t v, __nv_bfloat16) {
  return (double)__uint_as_float(v << 16);
}
__device__ __forceinline__ double widen_hi(uint32_t v, __nv_bfloat16) {
  return (double)__uint_as_float(v & 0xFFFF0000u);
}

// Partial ||x||^2 (fp32) of one 16-bit row, summed in 64-element blocks until
// kFarRatioExactM1 times it reaches `lim2` (= -2 v): the full norm when the row
// is far, else a partial sum that already rules the row out (most rows stop
// after one block).  d % 8 == 0, 16-byte aligned rows.
template <typename T>
__device__ __forceinline__ float row_norm2_upto(const T *__restrict__ x, int d, float lim2) {
  const uint4 *xr = reinterpret_cast<const uint4 *>(x);
  const int n = d / 8;
  float s = 0.f;
  for (int j0 = 0; j0 < n && kFarRatioExactM1 * s < lim2; j0 += 8) {
    uint4 v[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) v[t] = j0 + t < n ? __ldg(xr + j0 + t) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const uint32_t w[4] = {v[t].x, v[t].y, v[t].z, v[t].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float lo = (float)widen_lo(w[q], T()), hi = (float)widen_hi(w[q], T());
        s = fmaf(lo, lo, s);
        s = fmaf(hi, hi, s);
      }
    }
  }
  return s;
}

// Exact nearest centroid of one point, computed by the whole warp: lane l
// takes centroids l, l + 32, ... and sums (x_j - c_kj)^2 over j in fp64 (the
// 16-bit inputs widen exactly); the lanes' (distance, k) pairs are then
// reduced to the smallest distance, lowest k on ties.  x: the point's row;
// c: its batch's (K, d) centroids; d % 8 == 0 and both 16-byte aligned.
template <typename T>
__device__ __noinline__ int exact_argmin_warp(const T *__restrict__ x, const T *__restrict__ c, int K,
                                              int d, int lane) {
  double best = __longlong_as_double(0x7ff0000000000000LL);  // +inf
  int bk = 0x7fffffff;
  const uint4 *xr = reinterpret_cast<const uint4 *>(x);
  for (int k = lane; k < K; k += 32) {
    const uint4 *cr = reinterpret_cast<const uint4 *>(c + (size_t)k * d);
    double s = 0.0;
    for (int j = 0; j < d / 8; ++j) {
      const uint4 xv = __ldg(xr + j), cv = __ldg(cr + j);
      const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w}, cs[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const double e0 = widen_lo(xs[q], T()) - widen_lo(cs[q], T());
        s = fma(e0, e0, s);
        const double e1 = widen_hi(xs[q], T()) - widen_hi(cs[q], T());
        s = fma(e1, e1, s);
      }
    }
    if (s < best) {  // k grows along a lane: ties keep the lower k
      best = s;
      bk = k;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int ok = __shfl_xor_sync(0xffffffffu, bk, o);
    if (ob < best || (ob == best && ok < bk)) {
      best = ob;
      bk = ok;
    }
  }
  return bk;
}

// One MMA step of the element type's kind: kind::f16 for fp16 / bf16 (K = 16),
// kind::tf32 for fp32 (K = 8); either way 32 bytes of every operand row.
template <typename T>
__device__ __forceinline__ void mma_t(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                      uint32_t accumulate) {
  if constexpr (sizeof(T) == 4) sm100::mma_tf32(d_tmem, a_desc, b_desc, idesc, accumulate);
  else sm100::mma_f16(d_tmem, a_desc, b_desc, idesc, accumulate);
}

// Stores one 32-byte norm row at row r of a K-major 32-byte-swizzled tile:
// 16-byte chunk q of row r sits at r * 32 + ((q ^ ((r >> 2) & 1)) * 16).
__device__ __forceinline__ void store_row32_sw32(uint8_t *tile, int r, const void *row) {
  const int flip = (r >> 2) & 1;
  uint4 *p = reinterpret_cast<uint4 *>(tile + r * 32);
  p[flip] = reinterpret_cast<const uint4 *>(row)[0];
  p[flip ^ 1] = reinterpret_cast<const uint4 *>(row)[1];
}
template <typename T>
__device__ __forceinline__ void store_ext_row_sw32(uint8_t *tile, int r, const T (&row)[kExt]) {
  store_row32_sw32(tile, r, row);
}

// a0 += lo(v)^2, a1 += hi(v)^2 for two packed 16-bit values, fp32 accumulation
// (mixed-precision FMA: the 16-bit inputs are exact in fp32, one rounding).
template <typename T> __device__ __forceinline__ void sq2_acc(uint32_t v, float &a0, float &a1);
template <> __device__ __forceinline__ void sq2_acc<__half>(uint32_t v, float &a0, float &a1) {
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
      "fma.rn.f32.f16 %0, lo, lo, %0;\n\tfma.rn.f32.f16 %1, hi, hi, %1;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "r"(v));
}
template <> __device__ __forceinline__ void sq2_acc<__nv_bfloat16>(uint32_t v, float &a0, float &a1) {
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
      "fma.rn.f32.bf16 %0, lo, lo, %0;\n\tfma.rn.f32.bf16 %1, hi, hi, %1;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "r"(v));
}

// Running argmax over one 32-column TMEM load with packed keys: the low byte
// of each (negative) accumulator is replaced by its column (a byte taken from
// colb, which holds the bytes 0..127).  For negative floats a larger key means
// a smaller |acc|, and among equal upper bits the smaller column.  Four
// independent max chains.
__device__ __forceinline__ void scan_packed(const uint32_t (&r)[32], const uint32_t cb,
                                            const uint32_t (&colb)[32], float &m0, float &m1,
                                            float &m2, float &m3) {
#define FK_KEY(t) __uint_as_float(__byte_perm(r[j + (t)], colb[(cb + j + (t)) >> 2], 0x3214u + ((cb + j + (t)) & 3u)))
#pragma unroll
  for (int j = 0; j < 32; j += 8) {
    m0 = max3f(m0, FK_KEY(0), FK_KEY(1));
    m1 = max3f(m1, FK_KEY(2), FK_KEY(3));
    m2 = max3f(m2, FK_KEY(4), FK_KEY(5));
    m3 = max3f(m3, FK_KEY(6), FK_KEY(7));
  }
#undef FK_KEY
}

// Exact running argmax over one 32-column TMEM load: chain t sees columns
// j = t (mod 4) in increasing order and moves only on a strictly larger value.
__device__ __forceinline__ void scan_exact(const uint32_t (&r)[32], const int cb, float (&lb)[4],
                                           int (&li)[4]) {
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float v = __uint_as_float(r[j + t]);
      if (v > lb[t]) {
        lb[t] = v;
        li[t] = cb + j + t;
      }
    }
  }
}


}  // namespace fk
