// fp32 points on the tensor cores: operands for a 3xTF32 FlashAssign.
//
// kind::tf32 multiplies 32-bit values with 10 fraction bits.  Each value v is
// split into hi = v truncated to tf32 and lo = v - hi (exact in fp32), and
// the rows are widened to 3d values:
//   points     [hi | hi | lo]        centroids  [hi | lo | hi]
// so one FlashAssign pass over the extended rows accumulates
//   x_hi.c_hi + x_hi.c_lo + x_lo.c_hi = x.c - x_lo.c_lo (+ tf32 rounding of the lo parts)
// in fp32: the dot product to about 2^-21 relative, the precision the pages
// ask of the fp32 path ("large-D + fp32 ok": "flash-kmeans and the return of
// exact K-Means on the GPU", section "Exact K-Means, with the assignment step
// written in Triton").  ||c||^2 / 2 enters through the norm rows
// (fk_norms.cuh, tf32 rows) computed from the fp32 centroids.
#include "fk_internal.h"
#include "fk_norms.cuh"

namespace fk {
namespace {

// dst (rows, 3d) from src (rows, d), d % 4 == 0, four values per thread.
__global__ void __launch_bounds__(256) k_split3(const float4 *__restrict__ src, long long rows,
                                                int d4, float4 *__restrict__ dst, int centroids) {
  const long long n = rows * d4;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const long long r = e / d4;
    const int j = (int)(e - r * d4);
    const float4 v = __ldg(src + e);
    const float4 hi = make_float4(tf32_trunc(v.x), tf32_trunc(v.y), tf32_trunc(v.z), tf32_trunc(v.w));
    const float4 lo = make_float4(v.x - hi.x, v.y - hi.y, v.z - hi.z, v.w - hi.w);
    float4 *o = dst + r * 3 * d4 + j;
    o[0] = hi;
    o[d4] = centroids ? lo : hi;
    o[2 * d4] = centroids ? hi : lo;
  }
}

// Norm rows of the fp32 centroids: one warp per (batch, padded centroid),
// ||c||^2 in fp32 (lane-strided FMA, then a butterfly sum).
__global__ void __launch_bounds__(256) k_prep_ext_f32(const float *__restrict__ c, int B, int K, int d,
                                                      long long Kpad, float4 *__restrict__ cnx) {
  const long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= (long long)B * Kpad) return;
  const int b = (int)(w / Kpad), k = (int)(w % Kpad);
  float s = 0.f;
  if (k < K) {
    const float *row = c + ((size_t)b * K + k) * d;
    for (int j = lane; j < d; j += 32) s = fmaf(row[j], row[j], s);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  }
  if (lane == 0) {  // stored pre-swizzled, like the 16-bit rows (fk_centroids.cu)
    alignas(16) float row[kExtF32];
    ext_centroid_row_f32(s, k < K, row);
    const int flip = (int)((w >> 2) & 1);
    cnx[2 * w + flip] = *reinterpret_cast<const float4 *>(&row[0]);
    cnx[2 * w + (flip ^ 1)] = *reinterpret_cast<const float4 *>(&row[4]);
  }
}

}  // namespace

bool use_tf32(int K, int d) { return d % 4 == 0 && (long long)K * d >= kTf32MinKd; }

int launch_split3(const float *src, long long rows, int d, float *dst, bool centroids, cudaStream_t s) {
  const long long n = rows * (d / 4);
  long long blocks = (n + 255) / 256;
  const long long cap = (long long)num_sms() * 16;
  if (blocks > cap) blocks = cap;
  if (blocks == 0) return FK_OK;
  k_split3<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<const float4 *>(src), rows, d / 4,
                                            reinterpret_cast<float4 *>(dst), centroids ? 1 : 0);
  FK_TRY(launched());
  FK_CUDA(cudaGetLastError());
  return FK_OK;
}

int launch_prep_ext_f32(const float *c, int B, int K, int d, long long Kpad, void *cnx, cudaStream_t s) {
  const long long warps = (long long)B * Kpad;
  k_prep_ext_f32<<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(c, B, K, d, Kpad, static_cast<float4 *>(cnx));
  FK_TRY(launched());
  FK_CUDA(cudaGetLastError());
  return FK_OK;
}

}  // namespace fk
