// fp32 assign on CUDA cores.
//
// ids[b,i] = argmin_k sum_j (x[b,i,j] - c[b,k,j])^2 in fp32, lowest k on ties.
// The squared distance is evaluated directly (same argmin as ||c||^2 - 2 x.c,
// without its cancellation), one point per thread, centroids staged through
// shared memory in 32 x 32 tiles; no distance matrix is written
// ("flash-kmeans and the return of exact K-Means on the GPU", section "The
// point of the kernel is that the distance matrix never exists": centroids
// stream in chunks while each point keeps a running argmin).
#include "fk_internal.h"

namespace fk {
namespace {

constexpr int kThreads = 128;
constexpr int kKC = 32;  // centroids per smem tile
constexpr int kDC = 32;  // dimensions per smem tile

__global__ void __launch_bounds__(kThreads) k_assign_f32(const float *__restrict__ x,
                                                         const float *__restrict__ c, int N, int K,
                                                         int d, int32_t *__restrict__ ids) {
  __shared__ float cs[kKC][kDC + 1];
  const int b = blockIdx.y;
  const long long row = (long long)blockIdx.x * kThreads + threadIdx.x;
  const bool valid = row < N;
  const float *xr = x + ((size_t)b * N + (valid ? row : 0)) * d;
  const float *cb = c + (size_t)b * K * d;
  float best = __int_as_float(0x7f800000);
  int bidx = 0;
  for (int k0 = 0; k0 < K; k0 += kKC) {
    float acc[kKC];
#pragma unroll
    for (int t = 0; t < kKC; ++t) acc[t] = 0.f;
    for (int j0 = 0; j0 < d; j0 += kDC) {
      __syncthreads();
      for (int e = threadIdx.x; e < kKC * kDC; e += kThreads) {
        int kk = e / kDC, jj = e % kDC;
        int k = k0 + kk, j = j0 + jj;
        cs[kk][jj] = (k < K && j < d) ? cb[(size_t)k * d + j] : 0.f;
      }
      __syncthreads();
      float xs[kDC];
#pragma unroll
      for (int jj = 0; jj < kDC; ++jj) xs[jj] = (j0 + jj < d) ? xr[j0 + jj] : 0.f;
#pragma unroll
      for (int jj = 0; jj < kDC; ++jj) {
#pragma unroll
        for (int kk = 0; kk < kKC; ++kk) {
          float t = xs[jj] - cs[kk][jj];
          acc[kk] = fmaf(t, t, acc[kk]);
        }
      }
    }
#pragma unroll
    for (int kk = 0; kk < kKC; ++kk) {
      if (k0 + kk < K && acc[kk] < best) {
        best = acc[kk];
        bidx = k0 + kk;
      }
    }
  }
  if (valid) ids[(size_t)b * N + row] = bidx;
}

}  // namespace

int launch_assign_f32(const float *x, const float *c, int B, long long N, int K, int d,
                      int32_t *ids, cudaStream_t s) {
  dim3 grid((unsigned)((N + kThreads - 1) / kThreads), (unsigned)B);
  k_assign_f32<<<grid, kThreads, 0, s>>>(x, c, (int)N, K, d, ids);
  FK_TRY(launched());
  FK_CUDA(cudaGetLastError());
  return FK_OK;
}

}  // namespace fk
