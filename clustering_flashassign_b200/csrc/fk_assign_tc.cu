// FlashAssign on sm_100a tensor cores (step a1 for fp16 / bf16 inputs).
//
// ids[b,i] = argmin_k ( ||c_k||^2 - 2 x_i . c_k ), fp32 accumulation, lowest
// k on ties, without ever writing the (B, N, K) distance matrix
// ("Flash-KMeans: Fast and Memory-Efficient Exact K-Means", Abstract: the
// distance computation is fused with an online argmin; "flash-kmeans and the
// return of exact K-Means on the GPU", section "The point of the kernel is
// that the distance matrix never exists": point tiles and centroid chunks are
// streamed on chip and the cross term never leaves it).
//
// Mapping on a B200 SM (one persistent CTA per SM, 320 threads):
//   warp 0      TMA producer: point tiles (128 x d) and centroid chunks
//               (256 x 64 K-blocks) into 128-byte-swizzled shared memory,
//   warp 1      one thread issues tcgen05.mma (M=128, N=256, K=16, kind::f16)
//               into a TMEM accumulator; two accumulators (2 x 256 columns =
//               all 512 TMEM columns) let the MMA of chunk c+1 overlap the
//               epilogue of chunk c,
//   warps 2..9  epilogue: tcgen05.ld the 128 x 256 cross-term tile, add
//               ||c||^2 (v = cn - 2 acc, one FFMA), keep a running
//               (min, argmin) per point.  Two warps share each TMEM lane
//               quadrant and split the chunk's columns; their results are
//               combined once per point tile.
// Two variants, picked by d:
//   resident X (d <= 128): the point tile stays in shared memory for all K
//               chunks (double-buffered across tiles); only centroids stream.
//   split-d     (d > 128): each pipeline stage carries a 64-wide slice of the
//               point tile and the matching centroid slice; the d loop runs
//               inside each K chunk (the pages' split-D path, "flash-kmeans
//               and the return of exact K-Means on the GPU", section "The point
//               of the kernel ..." and "Unknown GPUs get a conservative
//               fallback").  The threshold is set by the shared-memory budget
//               of this design, not the pages' 512.
// Rows past N and centroid rows past K are zero-filled by TMA; padded
// centroid columns carry cn = +inf so they never win.
#include <cuda.h>

#include "fk_sm100.cuh"

namespace fk {
namespace {

using namespace sm100;

constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + kEpiWarps * 32;
constexpr uint32_t kXBlockBytes = kTileM * kBlockK * 2;   // 16 KB
constexpr uint32_t kCBlockBytes = kChunkN * kBlockK * 2;  // 32 KB
constexpr uint32_t kTmemCols = 512;

struct TcArgs {
  int N;
  int tiles_per_batch;
  int total_tiles;
  int nchunks;
  int kblocks;
  long long Kpad;
  const float *cn;
  int32_t *ids;
  int *err;
  uint32_t idesc;
};

template <bool RESIDENT, int KB, int STAGES>
struct Layout {
  static constexpr uint32_t kXBytes = RESIDENT ? 2u * KB * kXBlockBytes : 0u;
  static constexpr uint32_t kStageBytes = RESIDENT ? kCBlockBytes : kXBlockBytes + kCBlockBytes;
  static constexpr uint32_t kStagesOff = kXBytes;
  static constexpr uint32_t kBarOff = kStagesOff + STAGES * kStageBytes;
  // barriers: full[S], empty[S], xfull[2], xempty[2], accfull[2], accempty[2],
  //           mfull[2], mempty[2], drain
  static constexpr int kNumBars = 2 * STAGES + 13;
  static constexpr uint32_t kMiscOff = kBarOff + kNumBars * 8;       // tmem slot, abort flag
  static constexpr uint32_t kMergeOff = (kMiscOff + 16 + 15) / 16 * 16;
  static constexpr uint32_t kBytes = kMergeOff + 2 * kTileM * 8;
  static constexpr uint32_t kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
  static_assert(kAlloc <= 227 * 1024, "shared memory budget");
};

// Bounded wait that ignores the abort flag (teardown: let in-flight work land).
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity, int *err) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > kWaitLimitNs / 4) {
      atomicCAS(err, DEV_OK, DEV_TIMEOUT);
      return;
    }
  }
}

// Warp-uniform wait: lane 0 polls, the verdict is broadcast, and __syncwarp
// orders the other lanes' later reads after lane 0's acquire.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          int *err, int lane) {
  int r = 1;
  if (lane == 0) r = mbar_wait(bar, parity, abort_flag, err) ? 1 : 0;
  r = __shfl_sync(0xffffffffu, r, 0);
  __syncwarp();
  return r != 0;
}

template <bool RESIDENT, int KB, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    k_flash_assign(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmc,
                   const TcArgs a) {
  using L = Layout<RESIDENT, KB, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t x_base = sb;
  const uint32_t st_base = sb + L::kStagesOff;
  const uint32_t bar0 = sb + L::kBarOff;
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto xfull = [&](int i) { return bar0 + 8u * (2 * STAGES + i); };
  auto xempty = [&](int i) { return bar0 + 8u * (2 * STAGES + 2 + i); };
  auto accfull = [&](int i) { return bar0 + 8u * (2 * STAGES + 4 + i); };
  auto accempty = [&](int i) { return bar0 + 8u * (2 * STAGES + 6 + i); };
  auto mfull = [&](int i) { return bar0 + 8u * (2 * STAGES + 8 + i); };
  auto mempty = [&](int i) { return bar0 + 8u * (2 * STAGES + 10 + i); };
  const uint32_t drain = bar0 + 8u * (2 * STAGES + 12);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);
  float2 *merge = reinterpret_cast<float2 *>(smem + L::kMergeOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(xfull(i), 1);
      mbar_init(xempty(i), 1);
      mbar_init(accfull(i), 1);
      mbar_init(accempty(i), kEpiWarps);
      mbar_init(mfull(i), kEpiWarps / 2);
      mbar_init(mempty(i), kEpiWarps / 2);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmx);
    prefetch_tensormap(&tmc);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int kblocks = RESIDENT ? KB : a.kblocks;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t f = 0, g = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < a.total_tiles; tile += gridDim.x) {
        const int b = tile / a.tiles_per_batch;
        const int row0 = (tile % a.tiles_per_batch) * kTileM;
        if (RESIDENT) {
          const int xb = g & 1;
          if (!mbar_wait(xempty(xb), ((g >> 1) & 1) ^ 1, abort_flag, a.err)) { ok = false; break; }
          mbar_arrive_expect_tx(xfull(xb), KB * kXBlockBytes);
          for (int kb = 0; kb < KB; ++kb)
            tma_load_3d(&tmx, x_base + (xb * KB + kb) * kXBlockBytes, xfull(xb), kb * kBlockK, row0, b);
          ++g;
        }
        for (int c = 0; ok && c < a.nchunks; ++c) {
          for (int kb = 0; kb < kblocks; ++kb) {
            const int s = f % STAGES;
            if (!mbar_wait(empty(s), ((f / STAGES) & 1) ^ 1, abort_flag, a.err)) { ok = false; break; }
            const uint32_t dst = st_base + s * L::kStageBytes;
            if (RESIDENT) {
              mbar_arrive_expect_tx(full(s), kCBlockBytes);
              tma_load_3d(&tmc, dst, full(s), kb * kBlockK, c * kChunkN, b);
            } else {
              mbar_arrive_expect_tx(full(s), kXBlockBytes + kCBlockBytes);
              tma_load_3d(&tmx, dst, full(s), kb * kBlockK, row0, b);
              tma_load_3d(&tmc, dst + kXBlockBytes, full(s), kb * kBlockK, c * kChunkN, b);
            }
            ++f;
          }
        }
      }
      // tail: make every issued copy and every release of a stage land before exit
      const bool aborted = *abort_flag != 0;
      for (uint32_t ff = f > (uint32_t)STAGES ? f - STAGES : 0; ff < f; ++ff) {
        const int s = ff % STAGES;
        const uint32_t par = (ff / STAGES) & 1;
        wait_drain(aborted ? full(s) : empty(s), par, a.err);
      }
      if (RESIDENT) {
        for (uint32_t gg = g > 2 ? g - 2 : 0; gg < g; ++gg)
          wait_drain(aborted ? xfull(gg & 1) : xempty(gg & 1), (gg >> 1) & 1, a.err);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t f = 0, g = 0, h = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < a.total_tiles; tile += gridDim.x) {
        int xb = 0;
        if (RESIDENT) {
          xb = g & 1;
          if (!mbar_wait(xfull(xb), (g >> 1) & 1, abort_flag, a.err)) { ok = false; break; }
          tc_fence_after();
        }
        for (int c = 0; ok && c < a.nchunks; ++c) {
          const int ab = h & 1;
          if (!mbar_wait(accempty(ab), ((h >> 1) & 1) ^ 1, abort_flag, a.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem + ab * kChunkN;
          for (int kb = 0; kb < kblocks; ++kb) {
            const int s = f % STAGES;
            if (!mbar_wait(full(s), (f / STAGES) & 1, abort_flag, a.err)) { ok = false; break; }
            tc_fence_after();
            const uint32_t stage = st_base + s * L::kStageBytes;
            const uint32_t a_addr = RESIDENT ? x_base + (xb * KB + kb) * kXBlockBytes : stage;
            const uint32_t b_addr = RESIDENT ? stage : stage + kXBlockBytes;
#pragma unroll
            for (int k = 0; k < kBlockK / 16; ++k)
              mma_f16(d_tmem, desc_k_sw128(a_addr + k * 32), desc_k_sw128(b_addr + k * 32), a.idesc,
                      (kb | k) != 0 ? 1u : 0u);
            mma_commit(empty(s));  // frees the stage once these MMAs have read it
            ++f;
          }
          if (!ok) break;
          mma_commit(accfull(ab));  // accumulator ready for the epilogue
          ++h;
        }
        if (RESIDENT && ok) {
          mma_commit(xempty(xb));  // point tile no longer needed
          ++g;
        }
      }
      mma_commit(drain);  // arrives when every MMA issued above has completed
      wait_drain(drain, 0, a.err);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int quad = warp & 3;  // TMEM lanes this warp may read: 32 * (warp % 4) ...
    const int half = ew >> 2;   // which 128 columns of each chunk
    const int r_in_tile = quad * 32 + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16) + half * 128;
    uint32_t h = 0, u = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < a.total_tiles; tile += gridDim.x, ++u) {
      const int b = tile / a.tiles_per_batch;
      const int row0 = (tile % a.tiles_per_batch) * kTileM;
      const float *cnb = a.cn + (size_t)b * a.Kpad + half * 128;
      float best = __int_as_float(0x7f800000);
      int bidx = 0;
      for (int c = 0; c < a.nchunks; ++c, ++h) {
        const int ab = h & 1;
        if (!warp_wait(accfull(ab), (h >> 1) & 1, abort_flag, a.err, lane)) { ok = false; break; }
        tc_fence_after();
        const float *cnc = cnb + (size_t)c * kChunkN;
        float lb[4] = {best, best, best, best};
        int li[4] = {-1, -1, -1, -1};
#pragma unroll
        for (int gp = 0; gp < 2; ++gp) {
          uint32_t r0[32], r1[32];
          tmem_ld_32x32b_x32(t_lane + ab * kChunkN + gp * 64, r0);
          tmem_ld_32x32b_x32(t_lane + ab * kChunkN + gp * 64 + 32, r1);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const float4 cv = __ldg(reinterpret_cast<const float4 *>(cnc + gp * 64 + j));
            const float v0 = fmaf(__uint_as_float(r0[j + 0]), -2.f, cv.x);
            const float v1 = fmaf(__uint_as_float(r0[j + 1]), -2.f, cv.y);
            const float v2 = fmaf(__uint_as_float(r0[j + 2]), -2.f, cv.z);
            const float v3 = fmaf(__uint_as_float(r0[j + 3]), -2.f, cv.w);
            if (v0 < lb[0]) { lb[0] = v0; li[0] = gp * 64 + j + 0; }
            if (v1 < lb[1]) { lb[1] = v1; li[1] = gp * 64 + j + 1; }
            if (v2 < lb[2]) { lb[2] = v2; li[2] = gp * 64 + j + 2; }
            if (v3 < lb[3]) { lb[3] = v3; li[3] = gp * 64 + j + 3; }
          }
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const float4 cv = __ldg(reinterpret_cast<const float4 *>(cnc + gp * 64 + 32 + j));
            const float v0 = fmaf(__uint_as_float(r1[j + 0]), -2.f, cv.x);
            const float v1 = fmaf(__uint_as_float(r1[j + 1]), -2.f, cv.y);
            const float v2 = fmaf(__uint_as_float(r1[j + 2]), -2.f, cv.z);
            const float v3 = fmaf(__uint_as_float(r1[j + 3]), -2.f, cv.w);
            if (v0 < lb[0]) { lb[0] = v0; li[0] = gp * 64 + 32 + j + 0; }
            if (v1 < lb[1]) { lb[1] = v1; li[1] = gp * 64 + 32 + j + 1; }
            if (v2 < lb[2]) { lb[2] = v2; li[2] = gp * 64 + 32 + j + 2; }
            if (v3 < lb[3]) { lb[3] = v3; li[3] = gp * 64 + 32 + j + 3; }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(accempty(ab));  // accumulator may be overwritten
        // merge the four chains: smaller value, then lower column
        float m = lb[0];
        int mi = li[0];
#pragma unroll
        for (int t = 1; t < 4; ++t) {
          if (li[t] >= 0 && (mi < 0 || lb[t] < m || (lb[t] == m && li[t] < mi))) {
            m = lb[t];
            mi = li[t];
          }
        }
        if (mi >= 0) {  // strictly below the running best (chains start at it)
          best = m;
          bidx = c * kChunkN + half * 128 + mi;
        }
      }
      if (!ok) break;
      // combine the two column halves of each row: lower value, then lower index
      const int p = u & 1;
      const uint32_t vpar = (u >> 1) & 1;
      float2 *slot = merge + p * kTileM + r_in_tile;
      if (half == 1) {
        if (!warp_wait(mempty(p), vpar ^ 1, abort_flag, a.err, lane)) { ok = false; break; }
        *slot = make_float2(best, __int_as_float(bidx));
        __syncwarp();
        if (lane == 0) mbar_arrive(mfull(p));
      } else {
        if (!warp_wait(mfull(p), vpar, abort_flag, a.err, lane)) { ok = false; break; }
        const float2 o = *slot;
        __syncwarp();
        if (lane == 0) mbar_arrive(mempty(p));
        const float ob = o.x;
        const int oi = __float_as_int(o.y);
        if (ob < best || (ob == best && oi < bidx)) {
          best = ob;
          bidx = oi;
        }
        const int row = row0 + r_in_tile;
        if (row < a.N) a.ids[(size_t)b * a.N + row] = bidx;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int get_encoder(EncodeTiledFn *out) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    FK_CUDA(cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q));
    if (q != cudaDriverEntryPointSuccess || !p)
      return set_error(FK_ECUDA, "cuTensorMapEncodeTiled not available from the driver");
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  *out = fn;
  return FK_OK;
}

// (d, rows, B) tensor of 16-bit elements, box (64, box_rows, 1), 128-byte swizzle.
int encode_3d(CUtensorMap *map, const void *base, int dtype, int d, long long rows, int B,
              int box_rows) {
  EncodeTiledFn enc;
  FK_TRY(get_encoder(&enc));
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)B};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)rows * d * 2};
  cuuint32_t box[3] = {(cuuint32_t)kBlockK, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, dtype == FK_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                   3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(FK_ECUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)r));
  return FK_OK;
}

template <bool RESIDENT, int KB, int STAGES>
int launch_variant(const CUtensorMap &tmx, const CUtensorMap &tmc, const TcArgs &a, int grid,
                   cudaStream_t s) {
  using L = Layout<RESIDENT, KB, STAGES>;
  static bool attr = false;
  if (!attr) {
    FK_CUDA(cudaFuncSetAttribute(k_flash_assign<RESIDENT, KB, STAGES>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kAlloc));
    attr = true;
  }
  k_flash_assign<RESIDENT, KB, STAGES><<<grid, kThreads, L::kAlloc, s>>>(tmx, tmc, a);
  count_launch();
  FK_CUDA(cudaGetLastError());
  return FK_OK;
}

}  // namespace

int launch_assign_tc(const void *x, const void *ch, const float *cn, int dtype, int B, long long N,
                     int K, int d, long long Kpad, int32_t *ids, int *err, cudaStream_t s) {
  CUtensorMap tmx, tmc;
  FK_TRY(encode_3d(&tmx, x, dtype, d, N, B, kTileM));
  FK_TRY(encode_3d(&tmc, ch, dtype, d, K, B, kChunkN));
  TcArgs a;
  a.N = (int)N;
  a.tiles_per_batch = (int)((N + kTileM - 1) / kTileM);
  long long total = (long long)B * a.tiles_per_batch;
  if (total > 0x7fffffffLL) return set_error(FK_EUNSUPPORTED, "too many point tiles");
  a.total_tiles = (int)total;
  a.nchunks = (K + kChunkN - 1) / kChunkN;
  a.kblocks = (d + kBlockK - 1) / kBlockK;
  a.Kpad = Kpad;
  a.cn = cn;
  a.ids = ids;
  a.err = err;
  a.idesc = sm100::idesc_f16(dtype == FK_BF16 ? 1u : 0u, kTileM, kChunkN);
  int grid = num_sms();
  if (total < grid) grid = (int)total;
  if (a.kblocks == 1) return launch_variant<true, 1, 5>(tmx, tmc, a, grid, s);
  if (a.kblocks == 2) return launch_variant<true, 2, 4>(tmx, tmc, a, grid, s);
  return launch_variant<false, 1, 4>(tmx, tmc, a, grid, s);
}

}  // namespace fk
