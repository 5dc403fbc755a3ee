// Segment reduction of the sort-inverse update (step a5, before finalize).
//
// After the counting sort, equal ids are contiguous: kv[b][j] = (id, point)
// holds the id at sorted position j and the index of the point there.  The points are
// never moved; rows are gathered in sorted order and each run of equal ids is
// reduced on chip in fp32 ("Flash-KMeans: IO感知的精确K-Means", section
// "它攻克的兩大瓶頸": every thread block reduces a segment on chip and issues
// one atomic add per segment, so the atomics drop from O(N d) to
// O((K + N/B_N) d)).
//
// Work split: the sorted array of each batch is cut into pieces of kPiece
// positions and d into column blocks of 32 lanes x VEC elements; one warp owns
// one (batch, piece, column block), so a hot cluster spread over many pieces is
// reduced by many warps and the work stays balanced however skewed the
// cluster sizes are.  There are at most K + N / kPiece flushes per batch and
// column block, as on the pages -- but the flush here is a plain store, not an
// atomic add, which makes the result independent of scheduling:
//   - the piece holding the first position of a segment "owns" it and stores
//     its run's sum to sums[b][k];
//   - a piece whose first run continues a segment from the previous piece
//     stores that run's sum to first[b][piece];
//   - the finalize adds the owner's sum and the continuation sums of the
//     following pieces in piece order.
// Every stored value has exactly one writer and is combined in a fixed order,
// so repeated runs give bit-identical centroids, and the sums need no zeroing.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "fk_internal.h"

namespace fk {
namespace {

constexpr int kWarps = 8;
constexpr int kUnroll = 16;  // rows in flight per warp

template <typename T, int VEC> struct RowLoad;

template <> struct RowLoad<float, 4> {
  static __device__ __forceinline__ void load(const float *p, float (&v)[4]) {
    const float4 u = __ldg(reinterpret_cast<const float4 *>(p));
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
  }
};
template <> struct RowLoad<float, 1> {
  static __device__ __forceinline__ void load(const float *p, float (&v)[1]) { v[0] = __ldg(p); }
};

template <int VEC> __device__ __forceinline__ void store(float *dst, const float (&a)[VEC]);
template <> __device__ __forceinline__ void store<4>(float *dst, const float (&a)[4]) {
  *reinterpret_cast<float4 *>(dst) = make_float4(a[0], a[1], a[2], a[3]);
}
template <> __device__ __forceinline__ void store<1>(float *dst, const float (&a)[1]) { *dst = a[0]; }

template <typename T, int VEC>
__global__ void __launch_bounds__(kWarps * 32) k_segreduce(const T *__restrict__ x,
                                                           const int2 *__restrict__ kv, int N,
                                                           int K, int d, int pieces, int colblocks,
                                                           long long items, float *__restrict__ sums,
                                                           float *__restrict__ first) {
  const int lane = threadIdx.x & 31;
  const long long item = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  pdl_wait();
  pdl_trigger();
  if (item >= items) return;
  const int cb = (int)(item % colblocks);
  const long long rest = item / colblocks;
  const int piece = (int)(rest % pieces);
  const int b = (int)(rest / pieces);
  const int c0 = cb * 32 * VEC + lane * VEC;
  const bool active = c0 < d;
  const int j0 = piece * kPiece;
  const int j1 = min(N, j0 + kPiece);
  const int2 *kvb = kv + (size_t)b * N;
  const T *xb = x + (size_t)b * N * d + c0;
  float *sb = sums + (size_t)b * K * d + c0;
  float *fb = first + ((size_t)b * pieces + piece) * d + c0;
  const int prev = j0 > 0 ? kvb[j0 - 1].x : -1;

  float acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
  int cur = -1, start = j0;
#define FK_EMIT()                                                                  \
  do {                                                                             \
    if (cur >= 0 && active) {                                                      \
      if (start == j0 && cur == prev) store<VEC>(fb, acc); /* continuation */      \
      else store<VEC>(sb + (size_t)cur * d, acc);          /* this piece owns it */ \
    }                                                                              \
  } while (0)
  for (int jb = j0; jb < j1; jb += 32) {
    const int n = min(32, j1 - jb);
    const int2 p = lane < n ? kvb[jb + lane] : make_int2(-1, 0);
    int mk = p.x;
    const int mr = p.y;
    // ids must be in [0, K) and rows in [0, N); anything else (left behind by
    // an out-of-range caller id) is skipped
    if ((unsigned)mk >= (unsigned)K || (unsigned)mr >= (unsigned)N) mk = -1;
    for (int u = 0; u < n; u += kUnroll) {
      float v[kUnroll][VEC];
      int kk[kUnroll];
#pragma unroll
      for (int q = 0; q < kUnroll; ++q) {
        const int idx = (u + q) & 31;
        kk[q] = __shfl_sync(0xffffffffu, mk, idx);
        const int r = __shfl_sync(0xffffffffu, mr, idx);
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
            FK_EMIT();
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
            cur = kk[q];
            start = jb + u + q;
          }
#pragma unroll
          for (int e = 0; e < VEC; ++e) acc[e] += v[q][e];
        }
      }
    }
  }
  FK_EMIT();
#undef FK_EMIT
}

// 16-bit points: the piece's 128 sorted positions are gathered in batches of
// 16 row slices (128 elements = 256 bytes each) into a double-buffered
// shared-memory area with cp.async (16-byte copies that bypass L1): two
// batches (8 KB) per warp are in flight while the previous one is summed, and
// 24 warps per SM keep ~190 KB of gathers in flight.  Run boundaries are found
// once per 32 positions with a ballot, and each run is summed four rows at a
// time, so there is no per-row key test on the critical path.
constexpr int kRowsPerBatch = 16;
constexpr int kSliceBytes = 256;                        // 128 x 16-bit elements
constexpr int kBatches = kPiece / kRowsPerBatch;        // 8
constexpr int kKeyChunks = kPiece / 32;                 // 4
constexpr int kBufBytes = kRowsPerBatch * kSliceBytes;  // 4 KB per batch buffer
// the batch loop below pairs two batches per 32-position key chunk
static_assert(2 * kRowsPerBatch == 32, "k_segreduce16 assumes two 16-row batches per key chunk");

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool ok) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(ok ? 16 : 0)
               : "memory");
}

// Batch t of the piece: rows 16 (t % 2) .. +15 of key chunk t / 2.  Each lane
// issues 8 copies: row 2i + lane / 16 of the batch, 16-byte chunk lane % 16.
template <typename T>
__device__ __forceinline__ void issue_batch(uint32_t dst, const T *xb, int d, int col_base,
                                            int key, int row, int t, int lane) {
  const int q0 = (t & 1) * kRowsPerBatch;
#pragma unroll
  for (int i = 0; i < kRowsPerBatch / 2; ++i) {
    const int rib = 2 * i + (lane >> 4);
    const int chunk = lane & 15;
    const int k = __shfl_sync(0xffffffffu, key, q0 + rib);
    const int r = __shfl_sync(0xffffffffu, row, q0 + rib);
    const bool ok = k >= 0 && col_base + chunk * 8 < d;
    const T *src = ok ? xb + (size_t)r * d + col_base + chunk * 8 : xb;
    cp_async16(dst + rib * kSliceBytes + chunk * 16, src, ok);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// acc[c] += element c of the row slice (4 consecutive 16-bit elements): the
// mixed-precision add widens the 16-bit operand exactly and rounds the fp32
// sum once, so it equals a conversion followed by an fp32 add, in one
// instruction instead of two.
template <typename T> __device__ __forceinline__ void add_row(float (&acc)[4], const uint8_t *slice);
template <> __device__ __forceinline__ void add_row<__half>(float (&acc)[4], const uint8_t *slice) {
  const uint2 u = *reinterpret_cast<const uint2 *>(slice);
  asm("{\n\t.reg .f16 a0, a1, a2, a3;\n\t"
      "mov.b32 {a0, a1}, %4;\n\t"
      "mov.b32 {a2, a3}, %5;\n\t"
      "add.rn.f32.f16 %0, a0, %0;\n\t"
      "add.rn.f32.f16 %1, a1, %1;\n\t"
      "add.rn.f32.f16 %2, a2, %2;\n\t"
      "add.rn.f32.f16 %3, a3, %3;\n\t}"
      : "+f"(acc[0]), "+f"(acc[1]), "+f"(acc[2]), "+f"(acc[3])
      : "r"(u.x), "r"(u.y));
}
template <>
__device__ __forceinline__ void add_row<__nv_bfloat16>(float (&acc)[4], const uint8_t *slice) {
  const uint2 u = *reinterpret_cast<const uint2 *>(slice);
  asm("{\n\t.reg .b16 a0, a1, a2, a3;\n\t"
      "mov.b32 {a0, a1}, %4;\n\t"
      "mov.b32 {a2, a3}, %5;\n\t"
      "add.rn.f32.bf16 %0, a0, %0;\n\t"
      "add.rn.f32.bf16 %1, a1, %1;\n\t"
      "add.rn.f32.bf16 %2, a2, %2;\n\t"
      "add.rn.f32.bf16 %3, a3, %3;\n\t}"
      : "+f"(acc[0]), "+f"(acc[1]), "+f"(acc[2]), "+f"(acc[3])
      : "r"(u.x), "r"(u.y));
}

template <typename T>
__global__ void __launch_bounds__(kWarps * 32) k_segreduce16(const T *__restrict__ x,
                                                             const int2 *__restrict__ kv, int N,
                                                             int K, int d, int pieces, int colblocks,
                                                             long long items, float *__restrict__ sums,
                                                             float *__restrict__ first) {
  extern __shared__ __align__(16) uint8_t red_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long item = (long long)blockIdx.x * kWarps + warp;
  pdl_wait();
  pdl_trigger();
  if (item >= items) return;
  const int cb = (int)(item % colblocks);
  const long long rest = item / colblocks;
  const int piece = (int)(rest % pieces);
  const int b = (int)(rest / pieces);
  const int col_base = cb * 128;
  const int c0 = col_base + lane * 4;
  const bool active = c0 < d;
  const int j0 = piece * kPiece;
  const int j1 = min(N, j0 + kPiece);
  const int nb = (j1 - j0 + kRowsPerBatch - 1) / kRowsPerBatch;
  const int2 *kvb = kv + (size_t)b * N;
  const T *xb = x + (size_t)b * N * d;
  float *sb = sums + (size_t)b * K * d + c0;
  float *fb = first + ((size_t)b * pieces + piece) * d + c0;
  uint8_t *wbuf = red_smem + warp * 2 * kBufBytes;
  const uint32_t buf = static_cast<uint32_t>(__cvta_generic_to_shared(wbuf));

  // keys / rows of the piece: lane l holds positions j0 + 32 t + l
  int mk[kKeyChunks], mr[kKeyChunks];
#pragma unroll
  for (int t = 0; t < kKeyChunks; ++t) {
    const int j = j0 + 32 * t + lane;
    const int2 p = j < j1 ? kvb[j] : make_int2(-1, 0);
    mk[t] = p.x;
    mr[t] = p.y;
    // ids must be in [0, K) and rows in [0, N); anything else (left behind by
    // an out-of-range caller id) is skipped
    if ((unsigned)mk[t] >= (unsigned)K || (unsigned)mr[t] >= (unsigned)N) mk[t] = -1;
  }
  const int prev = j0 > 0 ? kvb[j0 - 1].x : -1;
  issue_batch<T>(buf, xb, d, col_base, mk[0], mr[0], 0, lane);
  if (nb > 1) issue_batch<T>(buf + kBufBytes, xb, d, col_base, mk[0], mr[0], 1, lane);

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  int cur = -1, start = j0;
  unsigned bounds = 0;
#pragma unroll
  for (int t = 0; t < kBatches; ++t) {
    if (t >= nb) break;
    const int kc = t >> 1;
    if ((t & 1) == 0) {
      // run starts inside this key chunk: position q starts a run when its key
      // differs from position q - 1 (q = 0 compares with the open run)
      const int before = __shfl_up_sync(0xffffffffu, mk[kc], 1);
      const int pk = lane == 0 ? cur : before;
      bounds = __ballot_sync(0xffffffffu, mk[kc] != pk);
    }
    if (t + 1 < nb) asm volatile("cp.async.wait_group 1;" ::: "memory");
    else asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncwarp();
    const uint8_t *slab = wbuf + (t & 1) * kBufBytes + lane * 8;
    const int q0 = (t & 1) * kRowsPerBatch;
    const int qe = min(q0 + kRowsPerBatch, j1 - j0 - 32 * kc);
    int q = q0;
    while (q < qe) {
      // end of the run that contains position q
      const unsigned later = bounds & ~((2u << q) - 1u);
      const int e = min(qe, later ? __ffs(later) - 1 : 32);
      const int key = __shfl_sync(0xffffffffu, mk[kc], q);
      if (key != cur) {
        if (cur >= 0 && active) {
          if (start == j0 && cur == prev) store<4>(fb, acc);          // continuation
          else store<4>(sb + (size_t)cur * d, acc);                    // this piece owns it
        }
        acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
        cur = key;
        start = j0 + 32 * kc + q;
      }
      if (key >= 0 && active) {
        // even rows of the run into acc, odd rows into a2 (two short chains)
        float a2[4] = {0.f, 0.f, 0.f, 0.f};
        int r = q;
        for (; r + 2 <= e; r += 2) {
          add_row<T>(acc, slab + (r - q0) * kSliceBytes);
          add_row<T>(a2, slab + (r + 1 - q0) * kSliceBytes);
        }
        if (r < e) add_row<T>(acc, slab + (r - q0) * kSliceBytes);
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[c] += a2[c];
      }
      q = e;
    }
    __syncwarp();
    if (t + 2 < nb)
      issue_batch<T>(buf + (t & 1) * kBufBytes, xb, d, col_base, mk[(t + 2) >> 1], mr[(t + 2) >> 1],
                     t + 2, lane);
  }
  if (cur >= 0 && active) {
    if (start == j0 && cur == prev) store<4>(fb, acc);
    else store<4>(sb + (size_t)cur * d, acc);
  }
}

template <typename T>
int launch16(const void *x, const int2 *kv, int B, int N, int K, int d, float *sums, float *first,
             cudaStream_t s) {
  const int shm = kWarps * 2 * kBufBytes;
  FK_TRY(set_smem_limit((const void *)k_segreduce16<T>, shm));
  const int pieces = (N + kPiece - 1) / kPiece;
  const int colblocks = (d + 127) / 128;
  const long long items = (long long)B * pieces * colblocks;
  const unsigned grid = (unsigned)((items + kWarps - 1) / kWarps);
  FK_CUDA(launch_pdl(k_segreduce16<T>, dim3(grid), dim3(kWarps * 32), shm, s, (const T *)x, kv, N, K, d,
                     pieces, colblocks, items, sums, first));
  FK_TRY(launched());
  return FK_OK;
}

template <typename T, int VEC>
int launch(const void *x, const int2 *kv, int B, int N, int K, int d, float *sums, float *first,
           cudaStream_t s) {
  const int pieces = (N + kPiece - 1) / kPiece;
  const int colblocks = (d + 32 * VEC - 1) / (32 * VEC);
  const long long items = (long long)B * pieces * colblocks;
  const unsigned grid = (unsigned)((items + kWarps - 1) / kWarps);
  FK_CUDA(launch_pdl(k_segreduce<T, VEC>, dim3(grid), dim3(kWarps * 32), 0, s, (const T *)x, kv, N, K, d,
                     pieces, colblocks, items, sums, first));
  FK_TRY(launched());
  return FK_OK;
}

}  // namespace

int launch_segreduce(const void *x, int dtype, const int2 *kv, int B, long long N, int K, int d,
                     float *sums, float *first, cudaStream_t s) {
  if (dtype == FK_F16) return launch16<__half>(x, kv, B, (int)N, K, d, sums, first, s);
  if (dtype == FK_BF16) return launch16<__nv_bfloat16>(x, kv, B, (int)N, K, d, sums, first, s);
  if (d % 4 == 0) return launch<float, 4>(x, kv, B, (int)N, K, d, sums, first, s);
  return launch<float, 1>(x, kv, B, (int)N, K, d, sums, first, s);
}

}  // namespace fk
