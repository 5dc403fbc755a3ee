// Segment reduction of the sort-inverse update (step a5, before finalize).
//
// After the counting sort, equal ids are contiguous: skeys[b][j] is the id at
// sorted position j and perm[b][j] the point index there.  The points are
// never moved; rows are gathered in sorted order, summed in fp32 on chip, and
// each run of equal ids is flushed with one vector atomic add
// ("Flash-KMeans: IO感知的精确K-Means", section "它攻克的兩大瓶頸": every
// thread block reduces a segment on chip and issues one atomic add per
// segment, cutting atomics from O(N d) to O((K + N/B_N) d)).
//
// Work split: the sorted array of each batch is cut into fixed pieces of
// kPiece positions, and d into column blocks of 32 lanes x VEC elements.  One
// warp owns one (batch, piece, column block): a hot cluster spread over many
// pieces is reduced by many warps, so the work stays balanced however skewed
// the cluster sizes are.  A warp flushes at every id change inside its piece
// and at the piece end, so there are at most K + N / kPiece flushes per batch
// and column block.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fk_internal.h"

namespace fk {
namespace {

constexpr int kWarps = 8;
constexpr int kUnroll = 8;  // rows in flight per warp

template <typename T, int VEC> struct RowLoad;

// 16-bit types: 4 elements = 8 bytes per lane.
template <> struct RowLoad<__half, 4> {
  static __device__ __forceinline__ void load(const __half *p, float (&v)[4]) {
    uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
    float2 a = __half22float2(*reinterpret_cast<__half2 *>(&u.x));
    float2 b = __half22float2(*reinterpret_cast<__half2 *>(&u.y));
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
  }
};
template <> struct RowLoad<__nv_bfloat16, 4> {
  static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&v)[4]) {
    uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
    float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u.x));
    float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u.y));
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
  }
};
template <> struct RowLoad<float, 4> {
  static __device__ __forceinline__ void load(const float *p, float (&v)[4]) {
    float4 u = __ldg(reinterpret_cast<const float4 *>(p));
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
  }
};
template <> struct RowLoad<float, 1> {
  static __device__ __forceinline__ void load(const float *p, float (&v)[1]) { v[0] = __ldg(p); }
};

template <int VEC> __device__ __forceinline__ void flush(float *dst, const float (&a)[VEC]);
template <> __device__ __forceinline__ void flush<4>(float *dst, const float (&a)[4]) {
  atomicAdd(reinterpret_cast<float4 *>(dst), make_float4(a[0], a[1], a[2], a[3]));
}
template <> __device__ __forceinline__ void flush<1>(float *dst, const float (&a)[1]) {
  atomicAdd(dst, a[0]);
}

template <typename T, int VEC>
__global__ void __launch_bounds__(kWarps * 32) k_segreduce(const T *__restrict__ x,
                                                           const int32_t *__restrict__ skeys,
                                                           const int32_t *__restrict__ perm, int N,
                                                           int K, int d, int pieces, int colblocks,
                                                           long long items, float *__restrict__ sums) {
  const int lane = threadIdx.x & 31;
  const long long item = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (item >= items) return;
  const int cb = (int)(item % colblocks);
  const long long rest = item / colblocks;
  const int piece = (int)(rest % pieces);
  const int b = (int)(rest / pieces);
  const int c0 = cb * 32 * VEC + lane * VEC;
  const bool active = c0 < d;
  const int j0 = piece * kPiece;
  const int j1 = min(N, j0 + kPiece);
  const int32_t *kb = skeys + (size_t)b * N;
  const int32_t *pb = perm + (size_t)b * N;
  const T *xb = x + (size_t)b * N * d + c0;
  float *sb = sums + (size_t)b * K * d + c0;

  float acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
  int cur = -1;  // no open segment yet
  for (int jb = j0; jb < j1; jb += 32) {
    const int n = min(32, j1 - jb);
    const int mk = lane < n ? kb[jb + lane] : -1;
    const int mr = lane < n ? pb[jb + lane] : 0;
    for (int u = 0; u < n; u += kUnroll) {
      float v[kUnroll][VEC];
      int kk[kUnroll];
#pragma unroll
      for (int q = 0; q < kUnroll; ++q) {
        const int idx = (u + q) & 31;
        kk[q] = __shfl_sync(0xffffffffu, mk, idx);
        const int r = __shfl_sync(0xffffffffu, mr, idx);
        // Only ids in [0, K) and rows in [0, N) are touched: a caller id out of
        // range leaves holes in the sorted arrays, and those are skipped here.
        if ((unsigned)kk[q] >= (unsigned)K || (unsigned)r >= (unsigned)N) kk[q] = -1;
        if (u + q < n && active && kk[q] >= 0) {
          RowLoad<T, VEC>::load(xb + (size_t)r * d, v[q]);
        } else {
#pragma unroll
          for (int e = 0; e < VEC; ++e) v[q][e] = 0.f;
        }
      }
#pragma unroll
      for (int q = 0; q < kUnroll; ++q) {
        if (u + q < n && kk[q] >= 0) {
          if (kk[q] != cur) {  // warp-uniform: every lane sees the same key
            if (active && cur >= 0) flush<VEC>(sb + (size_t)cur * d, acc);
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
            cur = kk[q];
          }
#pragma unroll
          for (int e = 0; e < VEC; ++e) acc[e] += v[q][e];
        }
      }
    }
  }
  if (active && cur >= 0) flush<VEC>(sb + (size_t)cur * d, acc);
}

template <typename T, int VEC>
int launch(const void *x, const int32_t *skeys, const int32_t *perm, int B, int N, int K, int d,
           float *sums, cudaStream_t s) {
  const int pieces = (N + kPiece - 1) / kPiece;
  const int colblocks = (d + 32 * VEC - 1) / (32 * VEC);
  const long long items = (long long)B * pieces * colblocks;
  const unsigned grid = (unsigned)((items + kWarps - 1) / kWarps);
  k_segreduce<T, VEC><<<grid, kWarps * 32, 0, s>>>((const T *)x, skeys, perm, N, K, d, pieces,
                                                   colblocks, items, sums);
  count_launch();
  FK_CUDA(cudaGetLastError());
  return FK_OK;
}

}  // namespace

int launch_segreduce(const void *x, int dtype, const int32_t *skeys, const int32_t *perm, int B,
                     long long N, int K, int d, float *sums, cudaStream_t s) {
  if (dtype == FK_F16) return launch<__half, 4>(x, skeys, perm, B, (int)N, K, d, sums, s);
  if (dtype == FK_BF16) return launch<__nv_bfloat16, 4>(x, skeys, perm, B, (int)N, K, d, sums, s);
  if (d % 4 == 0) return launch<float, 4>(x, skeys, perm, B, (int)N, K, d, sums, s);
  return launch<float, 1>(x, skeys, perm, B, (int)N, K, d, sums, s);
}

}  // namespace fk
