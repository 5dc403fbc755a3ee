// Centroid-side kernels: ||c||^2 preparation, fk_lloyd initialisation, the
// update's finalize step (mean, empty-cluster rule, shift, dtype copy) and the
// per-chunk accumulation of the streamed path.
//
// Update rule: each centroid becomes the mean of the points assigned to it
// ("Flash-KMeans: IO感知的精确K-Means", section "什么是 Flash-KMeans"); a
// cluster with no points keeps its previous centroid.  The shift that feeds
// the tol test of the functional API ("flash-kmeans and the return of exact
// K-Means on the GPU", section "Exact K-Means, with the assignment step
// written in Triton") is the L2 norm of new - old, maximised over b, k.
//
// Layout of the work: one warp per centroid; lane l handles elements
// 4l..4l+3, 4l+128.. (d % 4 == 0) or l, l+32, ... otherwise.  ||c||^2 is
// accumulated in that element order and then butterfly-reduced across lanes,
// identically in every kernel here, so the value the Lloyd loop fuses into its
// finalize equals the one fk_assign computes from the same dtype centroids.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fk_internal.h"
#include "fk_norms.cuh"

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

__device__ __forceinline__ uint16_t bits16(__half v) { return __half_as_ushort(v); }
__device__ __forceinline__ uint16_t bits16(__nv_bfloat16 v) { return __bfloat16_as_ushort(v); }
__device__ __forceinline__ uint16_t bits16(float) { return 0; }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr int kWarpsPerBlock = 8;

// Writes the tensor-core extension row of one centroid (see fk_norms.cuh);
// rows past K get the sentinel row.  A norm beyond the fp16 digits' range is
// recorded as DEV_RANGE in the device error word.  The rows are stored as the
// shared-memory image of a 32-byte-swizzled K-major tile (the two 16-byte
// halves of row w swap places when bit 2 of w is set), so the assign moves a
// chunk's 256 rows with one untiled bulk copy.
template <typename T>
__device__ __forceinline__ void store_ext(T *cnx, long long w, bool real, float cn, int *err) {
  if constexpr (sizeof(T) == 2) {
    alignas(16) T row[kExt];
    if (ext_centroid_row<T>(cn, real, row) && err) atomicCAS(err, DEV_OK, DEV_RANGE);
    uint4 *dst = reinterpret_cast<uint4 *>(cnx + (size_t)w * kExt);
    const int flip = (int)((w >> 2) & 1);
    dst[flip] = *reinterpret_cast<const uint4 *>(&row[0]);
    dst[flip ^ 1] = *reinterpret_cast<const uint4 *>(&row[8]);
  } else {
    (void)cnx; (void)w; (void)real; (void)cn; (void)err;
  }
}

// Element loop shared by every kernel: f(j, n) handles elements j .. j+n-1.
template <bool V4, typename F>
__device__ __forceinline__ void for_lane_elems(int d, int lane, F &&f) {
  if (V4) {
    for (int j = lane * 4; j < d; j += 128) f(j, 4);
  } else {
    for (int j = lane; j < d; j += 32) f(j, 1);
  }
}

template <typename T, bool V4>
__global__ void k_prep_cn(const T *__restrict__ c, int B, int K, int d, long long Kpad,
                          T *__restrict__ cnx, int *err) {
  const long long w = (long long)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= (long long)B * Kpad) return;
  const int b = (int)(w / Kpad), k = (int)(w % Kpad);
  if (k >= K) {
    if (lane == 0) store_ext<T>(cnx, w, false, 0.f, err);
    return;
  }
  const T *row = c + ((size_t)b * K + k) * d;
  float s = 0.f;
  for_lane_elems<V4>(d, lane, [&](int j, int n) {
    for (int e = 0; e < n; ++e) {
      const float v = to_f<T>(row[j + e]);
      s = fmaf(v, v, s);
    }
  });
  s = warp_sum(s);
  if (lane == 0) store_ext<T>(cnx, w, true, s, err);
}

template <typename T, bool V4>
__global__ void k_init(const T *__restrict__ init, int B, int K, int d, long long Kpad,
                       float *__restrict__ master, T *__restrict__ ch, T *__restrict__ cnx,
                       int *err) {
  const long long w = (long long)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= (long long)B * Kpad) return;
  const int b = (int)(w / Kpad), k = (int)(w % Kpad);
  if (k >= K) {
    if (lane == 0 && cnx) store_ext<T>(cnx, w, false, 0.f, err);
    return;
  }
  const size_t off = ((size_t)b * K + k) * d;
  float s = 0.f;
  for_lane_elems<V4>(d, lane, [&](int j, int n) {
    for (int e = 0; e < n; ++e) {
      const T v = init[off + j + e];
      const float f = to_f<T>(v);
      master[off + j + e] = f;
      if (ch) ch[off + j + e] = v;
      s = fmaf(f, f, s);
    }
  });
  s = warp_sum(s);
  if (lane == 0 && cnx) store_ext<T>(cnx, w, true, s, err);
}

// Sum of cluster w: the owner piece's partial plus the continuation partials
// of the following pieces, in piece order (see fk_reduce.cu).
template <bool FROM_PIECES>
__device__ __forceinline__ float seg_sum(const float *sums, const float *first, size_t w_off,
                                         size_t first_b, int d, int p0, int pl, int j) {
  float s = sums[w_off + j];
  if (FROM_PIECES)
    for (int p = p0 + 1; p <= pl; ++p) s += first[first_b + (size_t)p * d + j];
  return s;
}

// One warp per centroid (no grid-stride loop, so every centroid's loads are
// in flight at once); held to 32 registers so that eight CTAs (64 warps)
// share an SM: the kernel waits on loads, and more warps hide more of them.  With d % 4 == 0 lane l handles elements 4l..4l+3,
// 4l+128.. with 16-byte loads and stores; the arithmetic order per element is
// the same as in the scalar form.
template <typename T, bool V4, bool FROM_PIECES>
__global__ void __launch_bounds__(kWarpsPerBlock * 32, 8)
    k_finalize(const float *__restrict__ sums, const float *__restrict__ first, int pieces,
               const int32_t *__restrict__ counts, const int32_t *__restrict__ offsets,
               float *__restrict__ centers, T *__restrict__ ch, T *__restrict__ cnx, int B, int K,
               int d, long long Kpad, unsigned *__restrict__ maxshift, int *err) {
  __shared__ float wmax[kWarpsPerBlock];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long w = (long long)blockIdx.x * kWarpsPerBlock + warp;
  float my_max = 0.f;
  const bool live = w < (long long)B * K;
  int cnt = 0, off = 0;
  if (FROM_PIECES) {
    // launched dependent on the segment reduce (do_update): the counts and
    // offsets come from the sort, two or more launches back, so they are
    // complete once this grid runs and are read before the wait; the
    // partial sums are read after it
    if (live) {  // through L2 (.cg): no reliance on this SM's L1 holding nothing stale
      cnt = __ldcg(counts + w);
      off = __ldcg(offsets + w);
    }
    pdl_wait();
    pdl_trigger();
  } else if (live) {
    cnt = __ldg(counts + w);
  }
  if (live) {
    const int b = (int)(w / K), k = (int)(w % K);
    int p0 = 0, pl = -1;
    if (FROM_PIECES && cnt > 0) {
      p0 = off / kPiece;
      pl = (off + cnt - 1) / kPiece;
    }
    const size_t w_off = (size_t)w * d;
    const size_t first_b = (size_t)b * pieces * d;
    float shift2 = 0.f, nrm = 0.f;
    if (V4) {
      for (int j = lane * 4; j < d; j += 128) {
        const float4 old = *reinterpret_cast<const float4 *>(centers + w_off + j);
        float4 nv = old;
        if (cnt > 0) {
          float4 sm = __ldg(reinterpret_cast<const float4 *>(sums + w_off + j));
          if (FROM_PIECES)
            for (int p = p0 + 1; p <= pl; ++p) {
              const float4 f = __ldg(reinterpret_cast<const float4 *>(first + first_b + (size_t)p * d + j));
              sm.x += f.x;
              sm.y += f.y;
              sm.z += f.z;
              sm.w += f.w;
            }
          nv = make_float4(sm.x / (float)cnt, sm.y / (float)cnt, sm.z / (float)cnt, sm.w / (float)cnt);
        }
        const float o4[4] = {old.x, old.y, old.z, old.w};
        const float n4[4] = {nv.x, nv.y, nv.z, nv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float t = n4[e] - o4[e];
          shift2 = fmaf(t, t, shift2);
        }
        *reinterpret_cast<float4 *>(centers + w_off + j) = nv;
        if (ch) {
          if constexpr (sizeof(T) == 2) {
            uint32_t packed[2] = {0u, 0u};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const T r = from_f<T>(n4[e]);
              const float rf = to_f<T>(r);
              nrm = fmaf(rf, rf, nrm);
              packed[e >> 1] |= (uint32_t)bits16(r) << (16 * (e & 1));
            }
            *reinterpret_cast<uint2 *>(ch + w_off + j) = make_uint2(packed[0], packed[1]);
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const T r = from_f<T>(n4[e]);
              ch[w_off + j + e] = r;
              const float rf = to_f<T>(r);
              nrm = fmaf(rf, rf, nrm);
            }
          }
        }
      }
    } else {
      for_lane_elems<V4>(d, lane, [&](int j, int n) {
        for (int e = 0; e < n; ++e) {
          const float old = centers[w_off + j + e];
          float nv = old;
          if (cnt > 0) nv = seg_sum<FROM_PIECES>(sums, first, w_off, first_b, d, p0, pl, j + e) / (float)cnt;
          const float t = nv - old;
          shift2 = fmaf(t, t, shift2);
          centers[w_off + j + e] = nv;
          if (ch) {
            const T r = from_f<T>(nv);
            ch[w_off + j + e] = r;
            const float rf = to_f<T>(r);
            nrm = fmaf(rf, rf, nrm);
          }
        }
      });
    }
    shift2 = warp_sum(shift2);
    nrm = warp_sum(nrm);
    if (lane == 0 && cnx) store_ext<T>(cnx, (long long)b * Kpad + k, true, nrm, err);
    my_max = sqrtf(shift2);
  }
  if (lane == 0) wmax[warp] = my_max;
  __syncthreads();
  if (threadIdx.x == 0 && maxshift) {
    float m = 0.f;
    for (int i = 0; i < kWarpsPerBlock; ++i) m = fmaxf(m, wmax[i]);
    atomicMax(maxshift, __float_as_uint(m));  // non-negative floats order as unsigned ints
  }
}

// Per-cluster totals of the segment partials, grid (blocks, B).  overwrite:
// gsum[b][k] = the cluster's sum (zero for an empty cluster), the counts are
// already final; otherwise gsum[b][k] += it and gcounts[b][k] += counts[b][k]
// (the streamed path folds its chunks in order, so the totals are
// reproducible).
template <bool V4>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    k_accumulate(const float *__restrict__ sums, const float *__restrict__ first, int pieces,
                 const int32_t *__restrict__ counts, const int32_t *__restrict__ offsets, int K,
                 int d, float *__restrict__ gsum, int32_t *__restrict__ gcounts, int overwrite) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  sums += (size_t)b * K * d;
  first += (size_t)b * pieces * d;
  counts += (size_t)b * K;
  offsets += (size_t)b * K;
  gsum += (size_t)b * K * d;
  for (long long k = (long long)blockIdx.x * kWarpsPerBlock + warp; k < K;
       k += (long long)gridDim.x * kWarpsPerBlock) {
    const int cnt = counts[k];
    const size_t w_off = (size_t)k * d;
    if (cnt == 0) {
      if (overwrite)
        for_lane_elems<V4>(d, lane, [&](int j, int n) {
          for (int e = 0; e < n; ++e) gsum[w_off + j + e] = 0.f;
        });
      continue;
    }
    const int off = offsets[k];
    const int p0 = off / kPiece, pl = (off + cnt - 1) / kPiece;
    for_lane_elems<V4>(d, lane, [&](int j, int n) {
      for (int e = 0; e < n; ++e) {
        const float v = seg_sum<true>(sums, first, w_off, 0, d, p0, pl, j + e);
        gsum[w_off + j + e] = overwrite ? v : gsum[w_off + j + e] + v;
      }
    });
    if (!overwrite && lane == 0) gcounts[(size_t)b * K + k] += cnt;
  }
}

inline unsigned blocks_for(long long warps) {
  return (unsigned)((warps + kWarpsPerBlock - 1) / kWarpsPerBlock);
}

template <typename T>
int prep_t(const void *c, int B, int K, int d, long long Kpad, void *cnx, int *err, cudaStream_t s) {
  const unsigned g = blocks_for((long long)B * Kpad);
  if (d % 4 == 0) k_prep_cn<T, true><<<g, kWarpsPerBlock * 32, 0, s>>>((const T *)c, B, K, d, Kpad, (T *)cnx, err);
  else k_prep_cn<T, false><<<g, kWarpsPerBlock * 32, 0, s>>>((const T *)c, B, K, d, Kpad, (T *)cnx, err);
  FK_TRY(launched());
  FK_CUDA(cudaGetLastError());
  return FK_OK;
}

template <typename T>
int init_t(const void *init, int B, int K, int d, long long Kpad, float *master, void *ch,
           void *cnx, int *err, cudaStream_t s) {
  const unsigned g = blocks_for((long long)B * Kpad);
  if (d % 4 == 0)
    k_init<T, true><<<g, kWarpsPerBlock * 32, 0, s>>>((const T *)init, B, K, d, Kpad, master, (T *)ch, (T *)cnx, err);
  else
    k_init<T, false><<<g, kWarpsPerBlock * 32, 0, s>>>((const T *)init, B, K, d, Kpad, master, (T *)ch, (T *)cnx, err);
  FK_TRY(launched());
  FK_CUDA(cudaGetLastError());
  return FK_OK;
}

template <typename T, bool FP>
int fin_t(const float *sums, const float *first, int pieces, const int32_t *counts,
          const int32_t *offsets, float *centers, void *ch, void *cnx, int B, int K, int d,
          long long Kpad, unsigned *maxshift, int *err, cudaStream_t s) {
  const unsigned g = blocks_for((long long)B * K);
  // from pieces (do_update): a dependent launch after the segment reduce
  auto go = [&](auto kern) -> cudaError_t {
    if (FP)
      return launch_pdl(kern, dim3(g), dim3(kWarpsPerBlock * 32), 0, s, sums, first, pieces, counts, offsets,
                        centers, (T *)ch, (T *)cnx, B, K, d, Kpad, maxshift, err);
    kern<<<g, kWarpsPerBlock * 32, 0, s>>>(sums, first, pieces, counts, offsets, centers, (T *)ch, (T *)cnx, B,
                                           K, d, Kpad, maxshift, err);
    return cudaGetLastError();
  };
  FK_CUDA(d % 4 == 0 ? go(k_finalize<T, true, FP>) : go(k_finalize<T, false, FP>));
  FK_TRY(launched());
  return FK_OK;
}

}  // namespace

int launch_prep_cn(const void *c, int dtype, int B, int K, int d, long long Kpad, void *cnx,
                   int *err, cudaStream_t s) {
  if (dtype == FK_F16) return prep_t<__half>(c, B, K, d, Kpad, cnx, err, s);
  if (dtype == FK_BF16) return prep_t<__nv_bfloat16>(c, B, K, d, Kpad, cnx, err, s);
  return prep_t<float>(c, B, K, d, Kpad, cnx, err, s);
}

int launch_init_centers(const void *init, int dtype, int B, int K, int d, long long Kpad,
                        float *master, void *ch, void *cnx, int *err, cudaStream_t s) {
  if (dtype == FK_F16) return init_t<__half>(init, B, K, d, Kpad, master, ch, cnx, err, s);
  if (dtype == FK_BF16) return init_t<__nv_bfloat16>(init, B, K, d, Kpad, master, ch, cnx, err, s);
  return init_t<float>(init, B, K, d, Kpad, master, nullptr, nullptr, err, s);
}

int launch_finalize(const float *sums, const float *first, int pieces, const int32_t *counts,
                    const int32_t *offsets, float *centers, void *ch, void *cnx, int dtype, int B,
                    int K, int d, long long Kpad, unsigned *maxshift, bool from_pieces, int *err,
                    cudaStream_t s) {
  if (dtype == FK_F16)
    return from_pieces ? fin_t<__half, true>(sums, first, pieces, counts, offsets, centers, ch, cnx, B, K, d, Kpad, maxshift, err, s)
                       : fin_t<__half, false>(sums, first, pieces, counts, offsets, centers, ch, cnx, B, K, d, Kpad, maxshift, err, s);
  if (dtype == FK_BF16)
    return from_pieces ? fin_t<__nv_bfloat16, true>(sums, first, pieces, counts, offsets, centers, ch, cnx, B, K, d, Kpad, maxshift, err, s)
                       : fin_t<__nv_bfloat16, false>(sums, first, pieces, counts, offsets, centers, ch, cnx, B, K, d, Kpad, maxshift, err, s);
  return from_pieces ? fin_t<float, true>(sums, first, pieces, counts, offsets, centers, nullptr, nullptr, B, K, d, Kpad, maxshift, err, s)
                     : fin_t<float, false>(sums, first, pieces, counts, offsets, centers, nullptr, nullptr, B, K, d, Kpad, maxshift, err, s);
}

int launch_accumulate(const float *sums, const float *first, int pieces, const int32_t *counts,
                      const int32_t *offsets, int B, int K, int d, float *gsum, int32_t *gcounts,
                      bool overwrite, cudaStream_t s) {
  unsigned g = blocks_for(K);
  const unsigned cap = (unsigned)num_sms() * 8;
  if (g > cap) g = cap;
  const dim3 grid(g, (unsigned)B);
  if (d % 4 == 0)
    k_accumulate<true><<<grid, kWarpsPerBlock * 32, 0, s>>>(sums, first, pieces, counts, offsets, K, d, gsum,
                                                            gcounts, overwrite ? 1 : 0);
  else
    k_accumulate<false><<<grid, kWarpsPerBlock * 32, 0, s>>>(sums, first, pieces, counts, offsets, K, d, gsum,
                                                             gcounts, overwrite ? 1 : 0);
  FK_TRY(launched());
  FK_CUDA(cudaGetLastError());
  return FK_OK;
}

}  // namespace fk
