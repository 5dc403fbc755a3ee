// Centroid-side kernels: ||c||^2 preparation, fk_lloyd initialisation and the
// update's finalize step (mean, empty-cluster rule, shift, dtype copy).
//
// Update rule: each centroid becomes the mean of the points assigned to it
// ("Flash-KMeans: IO感知的精确K-Means", section "什么是 Flash-KMeans"); a
// cluster with no points keeps its previous centroid.  The shift that feeds
// the tol test of the functional API ("flash-kmeans and the return of exact
// K-Means on the GPU", section "Exact K-Means, with the assignment step
// written in Triton") is the L2 norm of new - old, maximised over b, k.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fk_internal.h"

namespace fk {
namespace {

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__half>(__half v) { return __half2float(v); }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __half from_f<__half>(float v) { return __float2half_rn(v); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr int kWarpsPerBlock = 8;

// One warp per centroid.  cn from the stored (already rounded) values.
template <typename T>
__global__ void k_prep_cn(const T *__restrict__ c, int B, int K, int d, long long Kpad,
                          float *__restrict__ cn) {
  long long w = (long long)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  int lane = threadIdx.x & 31;
  long long total = (long long)B * Kpad;
  if (w >= total) return;
  int b = (int)(w / Kpad);
  int k = (int)(w % Kpad);
  if (k >= K) {
    if (lane == 0) cn[w] = __int_as_float(0x7f800000);  // +inf: padded columns never win
    return;
  }
  const T *row = c + ((size_t)b * K + k) * d;
  float s = 0.f;
  for (int j = lane; j < d; j += 32) {
    float v = to_f<T>(row[j]);
    s = fmaf(v, v, s);
  }
  s = warp_sum(s);
  if (lane == 0) cn[w] = s;
}

template <typename T>
__global__ void k_init(const T *__restrict__ init, int B, int K, int d, long long Kpad,
                       float *__restrict__ master, T *__restrict__ ch, float *__restrict__ cn) {
  long long w = (long long)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  int lane = threadIdx.x & 31;
  long long total = (long long)B * Kpad;
  if (w >= total) return;
  int b = (int)(w / Kpad);
  int k = (int)(w % Kpad);
  if (k >= K) {
    if (lane == 0 && cn) cn[w] = __int_as_float(0x7f800000);
    return;
  }
  size_t off = ((size_t)b * K + k) * d;
  float s = 0.f;
  for (int j = lane; j < d; j += 32) {
    T v = init[off + j];
    float f = to_f<T>(v);
    master[off + j] = f;
    if (ch) ch[off + j] = v;
    s = fmaf(f, f, s);
  }
  s = warp_sum(s);
  if (lane == 0 && cn) cn[w] = s;
}

// One warp per centroid: divide, keep empty clusters, shift, dtype copy, cn,
// and clear the sums for the next accumulation.
template <typename T>
__global__ void k_finalize(float *__restrict__ sums, const int32_t *__restrict__ counts,
                           float *__restrict__ centers, T *__restrict__ ch, float *__restrict__ cn,
                           int B, int K, int d, long long Kpad, unsigned *__restrict__ maxshift) {
  long long w = (long long)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  int lane = threadIdx.x & 31;
  if (w >= (long long)B * K) return;
  int b = (int)(w / K);
  int k = (int)(w % K);
  int cnt = counts[w];
  size_t off = (size_t)w * d;
  float shift2 = 0.f, nrm = 0.f;
  for (int j = lane; j < d; j += 32) {
    float old = centers[off + j];
    float s = sums[off + j];
    float nv = cnt > 0 ? s / (float)cnt : old;
    float t = nv - old;
    shift2 = fmaf(t, t, shift2);
    centers[off + j] = nv;
    sums[off + j] = 0.f;
    if (ch) {
      T r = from_f<T>(nv);
      ch[off + j] = r;
      float rf = to_f<T>(r);
      nrm = fmaf(rf, rf, nrm);
    }
  }
  shift2 = warp_sum(shift2);
  nrm = warp_sum(nrm);
  if (lane == 0) {
    if (cn) cn[(size_t)b * Kpad + k] = nrm;
    if (maxshift) atomicMax(maxshift, __float_as_uint(sqrtf(shift2)));
  }
}

inline unsigned blocks_for(long long warps) {
  return (unsigned)((warps + kWarpsPerBlock - 1) / kWarpsPerBlock);
}

}  // namespace

int launch_prep_cn(const void *c, int dtype, int B, int K, int d, long long Kpad, float *cn,
                   cudaStream_t s) {
  long long warps = (long long)B * Kpad;
  if (dtype == FK_F16)
    k_prep_cn<__half><<<blocks_for(warps), kWarpsPerBlock * 32, 0, s>>>((const __half *)c, B, K, d, Kpad, cn);
  else if (dtype == FK_BF16)
    k_prep_cn<__nv_bfloat16><<<blocks_for(warps), kWarpsPerBlock * 32, 0, s>>>((const __nv_bfloat16 *)c, B, K, d, Kpad, cn);
  else
    k_prep_cn<float><<<blocks_for(warps), kWarpsPerBlock * 32, 0, s>>>((const float *)c, B, K, d, Kpad, cn);
  count_launch();
  FK_CUDA(cudaGetLastError());
  return FK_OK;
}

int launch_init_centers(const void *init, int dtype, int B, int K, int d, long long Kpad,
                        float *master, void *ch, float *cn, cudaStream_t s) {
  long long warps = (long long)B * Kpad;
  if (dtype == FK_F16)
    k_init<__half><<<blocks_for(warps), kWarpsPerBlock * 32, 0, s>>>((const __half *)init, B, K, d, Kpad, master, (__half *)ch, cn);
  else if (dtype == FK_BF16)
    k_init<__nv_bfloat16><<<blocks_for(warps), kWarpsPerBlock * 32, 0, s>>>((const __nv_bfloat16 *)init, B, K, d, Kpad, master, (__nv_bfloat16 *)ch, cn);
  else
    k_init<float><<<blocks_for(warps), kWarpsPerBlock * 32, 0, s>>>((const float *)init, B, K, d, Kpad, master, nullptr, cn);
  count_launch();
  FK_CUDA(cudaGetLastError());
  return FK_OK;
}

int launch_finalize(float *sums, const int32_t *counts, float *centers, void *ch, float *cn,
                    int dtype, int B, int K, int d, long long Kpad, unsigned *maxshift,
                    cudaStream_t s) {
  long long warps = (long long)B * K;
  if (dtype == FK_F16)
    k_finalize<__half><<<blocks_for(warps), kWarpsPerBlock * 32, 0, s>>>(sums, counts, centers, (__half *)ch, cn, B, K, d, Kpad, maxshift);
  else if (dtype == FK_BF16)
    k_finalize<__nv_bfloat16><<<blocks_for(warps), kWarpsPerBlock * 32, 0, s>>>(sums, counts, centers, (__nv_bfloat16 *)ch, cn, B, K, d, Kpad, maxshift);
  else
    k_finalize<float><<<blocks_for(warps), kWarpsPerBlock * 32, 0, s>>>(sums, counts, centers, nullptr, cn, B, K, d, Kpad, maxshift);
  count_launch();
  FK_CUDA(cudaGetLastError());
  return FK_OK;
}

}  // namespace fk
