// FlashAssign on sm_100a tensor cores (step a1 for fp16 / bf16 inputs, and
// for fp32 inputs as 3xTF32 on extended rows built by fk_tf32.cu).
//
// ids[b,i] = argmin_k ||x_i - c_k||^2, fp32 accumulation, lowest k on ties,
// without ever writing the (B, N, K) distance matrix ("Flash-KMeans: Fast and
// Memory-Efficient Exact K-Means", Abstract: the distance computation is fused
// with an online argmin; "flash-kmeans and the return of exact K-Means on the
// GPU", section "The point of the kernel is that the distance matrix never
// exists": point tiles and centroid chunks are streamed on chip and the cross
// term never leaves it).
//
// Mapping on a B200 SM (one persistent CTA per SM, 384 threads):
//   warp 0      TMA producer: centroid chunks (256 x 64 K-blocks) into
//               128-byte-swizzled shared memory and each chunk's norm rows
//               (256 x 16, 32-byte swizzle); split-d: the point tile's
//               K-blocks too,
//   warp 1      one thread issues tcgen05.mma (M=128, N=256, K=16, kind::f16)
//               into a TMEM accumulator; two accumulators (2 x 256 columns =
//               all 512 TMEM columns) let the MMA of chunk c+1 overlap the
//               epilogue of chunk c.  After the d loop of a chunk one more
//               K = 16 step multiplies the point and centroid norm rows
//               (fk_norms.cuh), so the accumulator already holds the ranking
//               value and the epilogue reads nothing but TMEM,
//   warps 2..9  epilogue: tcgen05.ld the 128 x 256 tile and keep a running
//               argmax per point.  Two warps share each TMEM lane quadrant
//               and split the chunk's columns; their results are combined
//               once per point tile,
//   warps 10-11 (resident variant) ||x||^2 of each point tile (rows 0..63
//               and 64..127), from the precomputed norms or the shared copy,
//               written as the tile's norm rows; warp 11's lane 0 also
//               requests the point tiles (128 x d), one tile ahead.
// In the resident variant the MMA thread waits per chunk for its accumulator
// (released by the epilogue) and for the stage, and commits once to the
// stage's empty barrier: the stage is free and the epilogue may read the
// accumulator; the producer waits for nothing else and runs ahead as far as
// the stages allow.  The
// centroids' norm rows are stored pre-swizzled (fk_centroids.cu) and arrive
// by one bulk copy per chunk: the TMA unit moves tiles row by row, and 256
// rows of 32 bytes cost it about as much as 256 rows of 128 bytes.
// Two variants, picked by d:
//   resident X (d <= 128): the point tile stays in shared memory for all K
//               chunks (double-buffered across tiles); only centroids stream.
//               acc = -(||x - c||^2 + 2^-10 ||x||^2) / 2 - 2^-14 < 0, so the
//               epilogue packs the column into the low byte of acc (one PRMT
//               per value) and keeps a three-input float max (half an
//               instruction per value).  Columns whose acc agree in all other
//               bits count as tied and the lowest column wins; that merges
//               values within 2^-15 of each other (relative).  Relative to
//               |acc| that is harmless while the nearest squared distance is
//               below 16 ||x||^2 (the merged values then lie within 5e-4 ||x||^2
//               of each other).  A point beyond that bound (far from every
//               centroid compared with its own norm, e.g. x = 0) is flagged at
//               the end of its tile and re-ranked exactly: one warp computes
//               sum_j (x_j - c_kj)^2 in fp64 for every k (lowest k on ties).
//   split-d     (d > 128): each pipeline stage carries a 64-wide slice of the
//               point tile and the matching centroid slice; the d loop runs
//               inside each K chunk (the pages' split-D path, "flash-kmeans
//               and the return of exact K-Means on the GPU", sections "The
//               point of the kernel ..." and "Unknown GPUs get a conservative
//               fallback").  acc = x.c - ||c||^2 / 2 and the epilogue keeps an
//               exact (value, column) argmax; its cost is spread over d / 64
//               K-blocks.  The threshold is set by the shared-memory budget of
//               this design, not the pages' 512.  Instantiated for fp32
//               elements too (kind::tf32, K = 8 per MMA: a 128-byte K-block row
//               holds 32 values, so layouts and stage sizes are unchanged).
//               With a keys buffer every (tile, chunk) pair is its own work
//               item, consecutive CTAs taking one tile's chunks so they share
//               its reads in L2; the chunks merge by a 64-bit atomicMax per
//               point and k_keys_to_ids writes the ids.  For 16-bit points
//               the fp32 rounding of acc is set by ||c||^2, so a point whose
//               nearest squared distance exceeds 64 ||x||^2 (||x||^2 from the
//               caller's precomputed norms, else read from its row) is
//               re-ranked exactly as above; when it is flagged in its best
//               chunk it is flagged in every chunk, so every work item
//               reports the exact id.
// Every role waits by polling its mbarriers without suspending (a suspended
// thread resumes hundreds of cycles after the phase completes, and the
// per-chunk hand-offs between the roles are on the tensor core's critical
// path); each wait still gives up after the time limit or on the CTA's abort.
// Rows past N and centroid rows past K are zero-filled by TMA; padded centroid
// columns carry a sentinel norm row (acc about -2^31 or below) so they never win.
#include <cuda.h>

#include "fk_assign_common.cuh"

namespace fk {
namespace {

using namespace sm100;

constexpr int kEpiWarps = 8;
constexpr int kNormWarp = 2 + kEpiWarps;
constexpr int kLoadWarp = kNormWarp + 1;  // resident: point-tile copies
constexpr int kThreads = 32 * (kLoadWarp + 1);
constexpr uint32_t kXBlockBytes = kTileM * kBlockK * 2;   // 16 KB
constexpr uint32_t kCBlockBytes = kChunkN * kBlockK * 2;  // 32 KB
constexpr uint32_t kAExtBytes = kTileM * kExt * 2;        // 4 KB of point norm rows
constexpr uint32_t kBExtBytes = kChunkN * kExt * 2;       // 8 KB of centroid norm rows
constexpr int kExtSlots = 2;
constexpr uint32_t kTmemCols = 512;

struct TcArgs {
  int N;
  int K;
  int tiles_per_batch;
  int total_tiles;
  int nchunks;
  int kblocks;
  const float *xn;  // ||x||^2 per point (B, N), or NULL: computed from the shared tile
  float *xn_out;    // nullable (resident, xn NULL): the computed norms are stored here too
  int32_t *ids;
  int *err;
  uint32_t idesc;
  // optional: the counting sort's tile histogram, H[b][row / 2048][id] += 1
  uint32_t *hist;
  int hist_tiles;
  // resident variant: the points and centroids in global memory (B, N, d) and
  // (B, K, d), read only by the exact re-rank of flagged points
  const void *xg;
  const void *cg;
  int d;
  // split-d only, optional: per-point packed (value, index) keys; then every
  // (tile, chunk) pair is its own work item and chunks merge by atomicMax
  unsigned long long *keys;
  // the centroids' extension rows: per (batch, chunk) the kBExtBytes
  // shared-memory image of the chunk's 32-byte-swizzled norm rows
  const uint8_t *cnx;
};

// (value, index) as one 64-bit key whose unsigned order is: larger value
// first, then lower index (the value bits mapped to an order-preserving uint).
__device__ __forceinline__ unsigned long long pack_argmax(float v, int idx) {
  const uint32_t u = __float_as_uint(v);
  const uint32_t o = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)o << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)idx);
}

template <bool RESIDENT, int KB, int STAGES>
struct Layout {
  static constexpr uint32_t kXBytes = RESIDENT ? 2u * KB * kXBlockBytes : 0u;
  static constexpr uint32_t kAExtOff = kXBytes;
  static constexpr uint32_t kAExtTotal = RESIDENT ? 2u * kAExtBytes : kAExtBytes;
  static constexpr uint32_t kBExtOff = kAExtOff + kAExtTotal;
  // resident: a stage holds a whole chunk (its KB centroid K-blocks and its
  // norm rows), so the MMA thread waits and commits once per chunk; split-d:
  // a stage holds one 64-wide K-block of points and centroids, and the norm
  // rows have their own ring.
  static constexpr int kRing = RESIDENT ? 0 : kExtSlots;
  static constexpr uint32_t kStagesOff = kBExtOff + kRing * kBExtBytes;
  static constexpr uint32_t kStageBytes =
      RESIDENT ? KB * kCBlockBytes + kBExtBytes : kXBlockBytes + kCBlockBytes;
  static constexpr uint32_t kBarOff = kStagesOff + STAGES * kStageBytes;
  // barriers: full[S], empty[S], efull[E], eempty[E], xfull[2], xempty[2],
  //           xnfull[2], accfull[2], accempty[2], mfull[4], mempty[4], drain,
  //           xnfree[2]
  static constexpr int kNumBars = 2 * STAGES + 2 * kExtSlots + 21;
  static constexpr uint32_t kMiscOff = kBarOff + kNumBars * 8;  // tmem slot, abort flag
  static constexpr uint32_t kMergeOff = (kMiscOff + 16 + 15) / 16 * 16;
  // resident: ||x||^2 of the rows of the two point-tile buffers, for the
  // epilogue's far-point check
  static constexpr uint32_t kXnOff = kMergeOff + kTileM * 16;
  static constexpr uint32_t kBytes = kXnOff + (RESIDENT ? 2 * kTileM * 4 : 0);
  static constexpr uint32_t kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
  static_assert(kStagesOff % 1024 == 0, "swizzled tiles need 1024-byte alignment");
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
  if (lane == 0) r = mbar_wait_spin(bar, parity, abort_flag, err) ? 1 : 0;
  r = __shfl_sync(0xffffffffu, r, 0);
  __syncwarp();
  return r != 0;
}

template <typename T, bool RESIDENT, int KB, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    k_flash_assign(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmc,
                   const TcArgs a) {
  using L = Layout<RESIDENT, KB, STAGES>;
  constexpr int kBlockE = 128 / (int)sizeof(T);  // elements per 128-byte K-block row
  static_assert(!RESIDENT || sizeof(T) == 2, "the resident-tile variant is for 16-bit points");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t x_base = sb;
  const uint32_t aext_base = sb + L::kAExtOff;
  const uint32_t bext_base = sb + L::kBExtOff;
  const uint32_t st_base = sb + L::kStagesOff;
  const uint32_t bar0 = sb + L::kBarOff;
  constexpr int kB2 = 2 * STAGES + 2 * kExtSlots;
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto efull = [&](int e) { return bar0 + 8u * (2 * STAGES + e); };
  auto eempty = [&](int e) { return bar0 + 8u * (2 * STAGES + kExtSlots + e); };
  auto xfull = [&](int i) { return bar0 + 8u * (kB2 + i); };
  auto xempty = [&](int i) { return bar0 + 8u * (kB2 + 2 + i); };
  auto xnfull = [&](int i) { return bar0 + 8u * (kB2 + 4 + i); };
  auto accfull = [&](int i) { return bar0 + 8u * (kB2 + 6 + i); };
  auto accempty = [&](int i) { return bar0 + 8u * (kB2 + 8 + i); };
  auto mfull = [&](int q) { return bar0 + 8u * (kB2 + 10 + q); };   // per TMEM lane quadrant
  auto mempty = [&](int q) { return bar0 + 8u * (kB2 + 14 + q); };
  const uint32_t drain = bar0 + 8u * (kB2 + 18);
  auto xnfree = [&](int i) { return bar0 + 8u * (kB2 + 19 + i); };
  float *xnorm_s = reinterpret_cast<float *>(smem + L::kXnOff);  // [2][kTileM], resident only
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);
  float4 *merge = reinterpret_cast<float4 *>(smem + L::kMergeOff);  // [kTileM]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int e = 0; e < kExtSlots; ++e) {
      mbar_init(efull(e), 1);
      mbar_init(eempty(e), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(xfull(i), 1);
      mbar_init(xempty(i), 1);
      mbar_init(xnfull(i), 2);  // the norm and loader warps' halves
      mbar_init(accfull(i), 1);
      mbar_init(accempty(i), kEpiWarps);

      mbar_init(xnfree(i), kEpiWarps / 2);
    }
    for (int q = 0; q < 4; ++q) {  // the two warps of a lane quadrant hand over their halves
      mbar_init(mfull(q), 1);
      mbar_init(mempty(q), 1);
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
  if (!RESIDENT && warp == kNormWarp) {
    // split-d: one constant point-side row (the -S_e that multiply ||c||^2's digits)
    if constexpr (sizeof(T) == 4) {
      alignas(16) float row[kExtF32];
      ext_point_row_f32(row);
      for (int r = lane; r < kTileM; r += 32) store_row32_sw32(smem + L::kAExtOff, r, row);
    } else {
      alignas(16) T row[kExt];
      ext_point_row<T, false>(0.f, row);
      for (int r = lane; r < kTileM; r += 32) store_ext_row_sw32<T>(smem + L::kAExtOff, r, row);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int kblocks = RESIDENT ? KB : a.kblocks;
  // the set-up above overlaps the previous kernel of the stream; everything
  // below may read what it wrote
  pdl_wait();
  // Work items: a point tile with all its chunks, or (split-d with keys) one
  // (tile, chunk) pair, consecutive CTAs taking consecutive chunks of one tile
  // so that they read its K-blocks at about the same time (shared in L2).
  const bool per_chunk = !RESIDENT && a.keys != nullptr;
  const int ntask = per_chunk ? a.total_tiles * a.nchunks : a.total_tiles;
  auto task_tile = [&](int t) { return per_chunk ? t / a.nchunks : t; };
  auto chunk_lo = [&](int t) { return per_chunk ? t % a.nchunks : 0; };
  auto chunk_hi = [&](int t) { return per_chunk ? t % a.nchunks + 1 : a.nchunks; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t f = 0, e = 0;  // stages, ext rows
      bool ok = true;
      for (int task = blockIdx.x; ok && task < ntask; task += gridDim.x) {
        const int tile = task_tile(task);
        const int b = tile / a.tiles_per_batch;
        const int row0 = (tile % a.tiles_per_batch) * kTileM;
        for (int c = chunk_lo(task); ok && c < chunk_hi(task); ++c) {
          if (RESIDENT) {  // the whole chunk and its norm rows in one stage
            // empty(s) is committed once per chunk by the MMA thread: the
            // stage is free and the epilogue may read the chunk's accumulator
            const int s = f % STAGES;
            if (!mbar_wait_spin(empty(s), ((f / STAGES) & 1) ^ 1, abort_flag, a.err)) { ok = false; break; }
            const uint32_t dst = st_base + s * L::kStageBytes;
            mbar_arrive_expect_tx(full(s), L::kStageBytes);
            for (int kb = 0; kb < KB; ++kb)
              tma_load_3d(&tmc, dst + kb * kCBlockBytes, full(s), kb * kBlockE, c * kChunkN, b);
            bulk_load(dst + KB * kCBlockBytes, a.cnx + ((size_t)b * a.nchunks + c) * kBExtBytes, kBExtBytes,
                      full(s));
            ++f;
          } else {  // this chunk's centroid norm rows (used by the chunk's last MMA step)
            const int es = e % kExtSlots;
            if (!mbar_wait_spin(eempty(es), ((e / kExtSlots) & 1) ^ 1, abort_flag, a.err)) { ok = false; break; }
            mbar_arrive_expect_tx(efull(es), kBExtBytes);
            bulk_load(bext_base + es * kBExtBytes, a.cnx + ((size_t)b * a.nchunks + c) * kBExtBytes, kBExtBytes,
                      efull(es));
            ++e;
          }
          for (int kb = 0; !RESIDENT && kb < kblocks; ++kb) {
            const int s = f % STAGES;
            if (!mbar_wait_spin(empty(s), ((f / STAGES) & 1) ^ 1, abort_flag, a.err)) { ok = false; break; }
            const uint32_t dst = st_base + s * L::kStageBytes;
            mbar_arrive_expect_tx(full(s), kXBlockBytes + kCBlockBytes);
            tma_load_3d(&tmx, dst, full(s), kb * kBlockE, row0, b);
            tma_load_3d(&tmc, dst + kXBlockBytes, full(s), kb * kBlockE, c * kChunkN, b);
            ++f;
          }
        }
      }
      // tail: make every issued copy and every release of a buffer land before exit
      const bool aborted = *abort_flag != 0;
      for (uint32_t ff = f > (uint32_t)STAGES ? f - STAGES : 0; ff < f; ++ff)
        wait_drain(aborted ? full(ff % STAGES) : empty(ff % STAGES), (ff / STAGES) & 1, a.err);
      for (uint32_t ee = e > (uint32_t)kExtSlots ? e - kExtSlots : 0; ee < e; ++ee)
        wait_drain(aborted ? efull(ee % kExtSlots) : eempty(ee % kExtSlots), (ee / kExtSlots) & 1, a.err);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t f = 0, g = 0, h = 0, e = 0;
      bool ok = true;
      for (int task = blockIdx.x; ok && task < ntask; task += gridDim.x) {
        int xb = 0;
        if (RESIDENT) {  // the point tile and its norm rows
          xb = g & 1;
          if (!mbar_wait_spin(xfull(xb), (g >> 1) & 1, abort_flag, a.err)) { ok = false; break; }
          if (!mbar_wait_spin(xnfull(xb), (g >> 1) & 1, abort_flag, a.err)) { ok = false; break; }
          tc_fence_after();
        }
        const uint32_t a_ext = aext_base + (RESIDENT ? xb * kAExtBytes : 0u);
        for (int c = chunk_lo(task); ok && c < chunk_hi(task); ++c) {
          const int ab = h & 1;
          if (RESIDENT) {
            // the accumulator is free (the epilogue's release of the chunk two
            // back) and the stage has landed; one commit per chunk to empty(s)
            // frees the stage and hands the accumulator to the epilogue
            const uint32_t d_tmem = tmem + ab * kChunkN;
            const int s = f % STAGES;
            if (!mbar_wait_spin(accempty(ab), ((h >> 1) & 1) ^ 1, abort_flag, a.err)) { ok = false; break; }
            if (!mbar_wait_spin(full(s), (f / STAGES) & 1, abort_flag, a.err)) { ok = false; break; }
            tc_fence_after();
            const uint32_t stage = st_base + s * L::kStageBytes;
#pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
              const uint32_t a_addr = x_base + (xb * KB + kb) * kXBlockBytes;
              const uint32_t b_addr = stage + kb * kCBlockBytes;
#pragma unroll
              for (int k = 0; k < kBlockK / 16; ++k)
                mma_t<T>(d_tmem, desc_k_sw128(a_addr + k * 32), desc_k_sw128(b_addr + k * 32), a.idesc,
                        (kb | k) != 0 ? 1u : 0u);
            }
            // the norm step: acc += A_ext . B_ext (fk_norms.cuh)
            mma_t<T>(d_tmem, desc_k_sw32(a_ext), desc_k_sw32(stage + KB * kCBlockBytes), a.idesc, 1u);
            mma_commit(empty(s));  // stage free, accumulator complete
            ++f;
            ++h;
            continue;
          }
          if (!mbar_wait_spin(accempty(ab), ((h >> 1) & 1) ^ 1, abort_flag, a.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem + ab * kChunkN;
          for (int kb = 0; kb < kblocks; ++kb) {
            const int s = f % STAGES;
            if (!mbar_wait_spin(full(s), (f / STAGES) & 1, abort_flag, a.err)) { ok = false; break; }
            tc_fence_after();
            const uint32_t stage = st_base + s * L::kStageBytes;
            const uint32_t a_addr = RESIDENT ? x_base + (xb * KB + kb) * kXBlockBytes : stage;
            const uint32_t b_addr = RESIDENT ? stage : stage + kXBlockBytes;
#pragma unroll
            for (int k = 0; k < kBlockK / 16; ++k)
              mma_t<T>(d_tmem, desc_k_sw128(a_addr + k * 32), desc_k_sw128(b_addr + k * 32), a.idesc,
                      (kb | k) != 0 ? 1u : 0u);
            mma_commit(empty(s));  // frees the stage once these MMAs have read it
            ++f;
          }
          if (!ok) break;
          // the norm step: acc += A_ext . B_ext (fk_norms.cuh)
          if (RESIDENT && c == 0) {
            if (!mbar_wait_spin(xnfull(xb), (g >> 1) & 1, abort_flag, a.err)) { ok = false; break; }
            tc_fence_after();
          }
          const int es = e % kExtSlots;
          if (!mbar_wait_spin(efull(es), (e / kExtSlots) & 1, abort_flag, a.err)) { ok = false; break; }
          tc_fence_after();
          mma_t<T>(d_tmem, desc_k_sw32(a_ext), desc_k_sw32(bext_base + es * kBExtBytes), a.idesc, 1u);
          mma_commit(eempty(es));
          ++e;
          mma_commit(accfull(ab));  // accumulator ready for the epilogue
          ++h;
        }
        if (RESIDENT && ok) {
          mma_commit(xempty(xb));  // point tile and its norm rows no longer needed
          ++g;
        }
      }
      mma_commit(drain);  // arrives when every MMA issued above has completed
      wait_drain(drain, 0, a.err);
    }
    __syncwarp();
  } else if (warp == kNormWarp || warp == kLoadWarp) {
    // ------------------------------------------------------------ point tiles and norms
    // (resident) The loader's lane 0 requests tile g into the buffer of tile
    // g - 2 as soon as that tile's MMAs are done, a whole tile ahead of its
    // use.  ||x||^2 of each tile (the point-side norm rows, and the norms for
    // the epilogue's far-point check) is split between the two warps, rows
    // 0..63 here and 64..127 in the loader, so a tile whose norms are summed
    // from its shared copy is ready in half the time.
    uint32_t issued_tiles = 0;  // loader lane 0: tiles requested
    if constexpr (RESIDENT) {
      constexpr int kQ = kTileM / 64;  // 32-row groups per warp
      const bool loader = warp == kLoadWarp;
      const int q0 = loader ? kQ : 0;
      uint32_t g = 0;
      for (int tile = blockIdx.x; tile < a.total_tiles; tile += gridDim.x, ++g) {
        const int xb = g & 1;
        const int b = tile / a.tiles_per_batch;
        const int row0 = (tile % a.tiles_per_batch) * kTileM;
        if (loader) {
          int issued = 1;
          if (lane == 0) {
            issued = mbar_wait_spin(xempty(xb), ((g >> 1) & 1) ^ 1, abort_flag, a.err) ? 1 : 0;
            if (issued) {
              mbar_arrive_expect_tx(xfull(xb), KB * kXBlockBytes);
              for (int kb = 0; kb < KB; ++kb)
                tma_load_3d(&tmx, x_base + (xb * KB + kb) * kXBlockBytes, xfull(xb), kb * kBlockE, row0, b);
            }
          }
          issued = __shfl_sync(0xffffffffu, issued, 0);
          if (!issued) break;
          if (lane == 0) ++issued_tiles;
        }
        float xn2[kQ];
        if (a.xn) {  // issued before the wait: the loads overlap it
#pragma unroll
          for (int q = 0; q < kQ; ++q) {
            const int row = row0 + (q0 + q) * 32 + lane;
            xn2[q] = row < a.N ? __ldg(a.xn + (size_t)b * a.N + row) : 0.f;
          }
        }
        if (!warp_wait(xfull(xb), (g >> 1) & 1, abort_flag, a.err, lane)) break;
        if (!a.xn) {
          // lane l sums rows l + 32 q of the swizzled tile (16-byte chunk j of
          // row r sits at chunk j ^ (r & 7); r & 7 == l & 7 here)
          float s0[kQ], s1[kQ];
#pragma unroll
          for (int q = 0; q < kQ; ++q) s0[q] = s1[q] = 0.f;
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            const uint8_t *blk = smem + (xb * KB + kb) * kXBlockBytes + (q0 * 32 + lane) * 128;
#pragma unroll 2
            for (int j = 0; j < 8; ++j) {
              const int off = (j ^ (lane & 7)) << 4;
              uint4 v[kQ];
#pragma unroll
              for (int q = 0; q < kQ; ++q) v[q] = *reinterpret_cast<const uint4 *>(blk + q * 32 * 128 + off);
#pragma unroll
              for (int q = 0; q < kQ; ++q) {
                sq2_acc<T>(v[q].x, s0[q], s1[q]);
                sq2_acc<T>(v[q].y, s0[q], s1[q]);
                sq2_acc<T>(v[q].z, s0[q], s1[q]);
                sq2_acc<T>(v[q].w, s0[q], s1[q]);
              }
            }
          }
#pragma unroll
          for (int q = 0; q < kQ; ++q) xn2[q] = s0[q] + s1[q];
          if (a.xn_out) {  // kept for later assigns of the same points
#pragma unroll
            for (int q = 0; q < kQ; ++q) {
              const int row = row0 + (q0 + q) * 32 + lane;
              if (row < a.N) a.xn_out[(size_t)b * a.N + row] = xn2[q];
            }
          }
        }
        bool clamped = false;
#pragma unroll
        for (int q = 0; q < kQ; ++q) {
          alignas(16) T row[kExt];
          clamped |= ext_point_row<T, true>(xn2[q], row);
          store_ext_row_sw32<T>(smem + L::kAExtOff + xb * kAExtBytes, (q0 + q) * 32 + lane, row);
        }
        if (clamped) atomicCAS(a.err, DEV_OK, DEV_RANGE);
        // the norms for the epilogue's far-point check, once the epilogue has
        // finished the tile that used this buffer before (two tiles back); the
        // epilogue reads them after xnfull, so tile g + 2 cannot complete xnfull
        // before tile g's norms are read
        if (!warp_wait(xnfree(xb), ((g >> 1) & 1) ^ 1, abort_flag, a.err, lane)) break;
#pragma unroll
        for (int q = 0; q < kQ; ++q) xnorm_s[xb * kTileM + (q0 + q) * 32 + lane] = xn2[q];
        fence_proxy_async_smem();  // generic-proxy writes -> tensor-core reads
        __syncwarp();
        if (lane == 0) mbar_arrive(xnfull(xb));
      }
    }
    if (RESIDENT && warp == kLoadWarp && lane == 0) {
      const uint32_t g = issued_tiles;
      // tail: the issued copies land (or are consumed) before exit
      const bool aborted = *abort_flag != 0;
      for (uint32_t gg = g > 2 ? g - 2 : 0; gg < g; ++gg)
        wait_drain(aborted ? xfull(gg & 1) : xempty(gg & 1), (gg >> 1) & 1, a.err);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int quad = warp & 3;  // TMEM lanes this warp may read: 32 * (warp % 4) ...
    const int half = ew >> 2;   // which 128 columns of each chunk
    const int r_in_tile = quad * 32 + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16) + half * 128;
    uint32_t colb[32];  // bytes 0..127, the column codes of the packed keys
#pragma unroll
    for (int i = 0; i < 32; ++i) colb[i] = 0x03020100u + 0x04040404u * i;
    uint32_t h = 0, u = 0;
    bool ok = true;
    for (int task = blockIdx.x; ok && task < ntask; task += gridDim.x, ++u) {
      const int tile = task_tile(task);
      const int b = tile / a.tiles_per_batch;
      const int row0 = (tile % a.tiles_per_batch) * kTileM;
      float best = __int_as_float(0xff800000);  // -inf
      int bidx = 0;                              // chunk (packed) or column (exact) of best
      float xn = 0.f;                            // ||x||^2 of this row (resident, half 1)
      for (int c = chunk_lo(task); c < chunk_hi(task); ++c, ++h) {
        const int ab = h & 1;
        // resident: the chunk's one commit (empty of its stage) marks the
        // accumulator complete; the barrier cannot run a phase ahead, since the
        // chunk STAGES later needs this warp's release of a later chunk first
        const bool got = RESIDENT ? warp_wait(empty(h % STAGES), (h / STAGES) & 1, abort_flag, a.err, lane)
                                  : warp_wait(accfull(ab), (h >> 1) & 1, abort_flag, a.err, lane);
        if (!got) { ok = false; break; }
        tc_fence_after();
        const uint32_t tb = t_lane + ab * kChunkN;
        uint32_t ra[32], rb[32], rc[32], rd[32];
        tmem_ld_32x32b_x32(tb, ra);
        tmem_ld_32x32b_x32(tb + 32, rb);
        tmem_wait_ld();
        tmem_ld_32x32b_x32(tb + 64, rc);  // in flight while ra, rb are scanned
        tmem_ld_32x32b_x32(tb + 96, rd);
        if (RESIDENT) {
          float m0 = best, m1 = best, m2 = best, m3 = best;
          scan_packed(ra, 0, colb, m0, m1, m2, m3);
          scan_packed(rb, 32, colb, m0, m1, m2, m3);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(accempty(ab));  // accumulator may be overwritten
          if (half == 1 && c == chunk_lo(task)) {
            // ||x||^2 for the far-point check (header), read once per tile by
            // the warps that do not write the ids, off the tile's critical
            // end; xnfull completed before this tile's first MMA, and waiting
            // on it orders the norm warp's stores before these reads
            if (!warp_wait(xnfull(u & 1), (u >> 1) & 1, abort_flag, a.err, lane)) { ok = false; break; }
            xn = xnorm_s[(u & 1) * kTileM + r_in_tile];
            __syncwarp();
            if (lane == 0) mbar_arrive(xnfree(u & 1));  // the norm warp may reuse the slot
          }
          scan_packed(rc, 64, colb, m0, m1, m2, m3);
          scan_packed(rd, 96, colb, m0, m1, m2, m3);
          const float m = fmaxf(max3f(m0, m1, m2), m3);
          // a later chunk must beat the running best in the upper bits
          if (key_hi(m) > key_hi(best)) {
            best = m;
            bidx = c;
          }
        } else {
          float lb[4] = {best, best, best, best};
          int li[4] = {-1, -1, -1, -1};
          scan_exact(ra, 0, lb, li);
          scan_exact(rb, 32, lb, li);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(accempty(ab));
          scan_exact(rc, 64, lb, li);
          scan_exact(rd, 96, lb, li);
          // merge the four chains: larger value, then lower column
          float m = lb[0];
          int mi = li[0];
#pragma unroll
          for (int t = 1; t < 4; ++t) {
            if (li[t] >= 0 && (mi < 0 || lb[t] > m || (lb[t] == m && li[t] < mi))) {
              m = lb[t];
              mi = li[t];
            }
          }
          if (mi >= 0) {  // strictly above the running best (chains start at it)
            best = m;
            bidx = c * kChunkN + half * 128 + mi;
          }
        }
      }
      if (!ok) break;
      float val;
      int idx;
      if (RESIDENT) {
        val = key_hi(best);
        idx = bidx * kChunkN + half * 128 + (int)(__float_as_uint(best) & ~kKeyMask);
      } else {
        val = best;
        idx = bidx;
      }
      // combine the two column halves of each row: larger value, then lower
      // index (one slot per row; the two warps of a lane quadrant hand over
      // through their own barriers, so each waits only for its partner, and
      // the half-1 warp writes a tile's slot a whole tile after the half-0
      // warp read the previous one)
      const uint32_t vpar = u & 1;
      float4 *slot = merge + r_in_tile;
      if (half == 1) {
        if (!warp_wait(mempty(quad), vpar ^ 1, abort_flag, a.err, lane)) { ok = false; break; }
        *slot = make_float4(val, __int_as_float(idx), xn, 0.f);
        __syncwarp();
        if (lane == 0) mbar_arrive(mfull(quad));
      } else {
        if (!warp_wait(mfull(quad), vpar, abort_flag, a.err, lane)) { ok = false; break; }
        const float4 o = *slot;
        __syncwarp();
        if (lane == 0) mbar_arrive(mempty(quad));
        const float ov = o.x;
        const int oi = __float_as_int(o.y);
        if (ov > val || (ov == val && oi < idx)) {  // the value travels too: the keys compare it
          val = ov;
          idx = oi;
        }
        const int row = row0 + r_in_tile;
        if constexpr (RESIDENT) {
          // far-point check (see the header): flagged rows of this warp are
          // re-ranked one after another by the whole warp
          unsigned flagged = __ballot_sync(0xffffffffu, row < a.N && -val > kFarRatioHalf * o.z);
          while (flagged) {
            const int src = __ffs(flagged) - 1;
            flagged &= flagged - 1;
            const int r = row0 + quad * 32 + src;
            const T *xrow = static_cast<const T *>(a.xg) + ((size_t)b * a.N + r) * a.d;
            const T *cb = static_cast<const T *>(a.cg) + (size_t)b * a.K * a.d;
            const int k = exact_argmin_warp<T>(xrow, cb, a.K, a.d, lane);
            if (lane == src) idx = k;
          }
        }
        if constexpr (!RESIDENT && sizeof(T) == 2) {
          // far-point check of the exact-value path (fk_assign_common.cuh):
          // rows with v < 0 take ||x||^2 from the precomputed norms, else
          // sum their row in global memory until it rules them out, and
          // those far from every centroid compared with it are re-ranked
          // exactly
          const bool maybe = row < a.N && val < 0.f;
          float xn2 = 0.f;
          if (maybe)
            xn2 = a.xn ? __ldg(a.xn + (size_t)b * a.N + row)
                       : row_norm2_upto<T>(static_cast<const T *>(a.xg) + ((size_t)b * a.N + row) * a.d, a.d,
                                           -2.f * val);
          unsigned flagged = __ballot_sync(0xffffffffu, maybe && kFarRatioExactM1 * xn2 < -2.f * val);
          while (flagged) {
            const int src = __ffs(flagged) - 1;
            flagged &= flagged - 1;
            const int r = row0 + quad * 32 + src;
            const T *xrow = static_cast<const T *>(a.xg) + ((size_t)b * a.N + r) * a.d;
            const T *cb = static_cast<const T *>(a.cg) + (size_t)b * a.K * a.d;
            const int k = exact_argmin_warp<T>(xrow, cb, a.K, a.d, lane);
            if (lane == src) idx = k;
          }
        }
        if (row < a.N && per_chunk) {  // this chunk's best; the chunks merge in the keys
          atomicMax(a.keys + (size_t)b * a.N + row, pack_argmax(val, idx));
        } else if (row < a.N) {
          a.ids[(size_t)b * a.N + row] = idx;
          if (a.hist)  // the sort's first kernel, fused: count the id in its sort tile
            atomicAdd(a.hist + ((size_t)b * a.hist_tiles + row / kSortTile) * a.K + idx, 1u);
        }
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

// Split-d with per-chunk work items: ids from the merged keys (and the
// sort's tile histogram, when fused), then the keys are cleared for the next
// launch.
__global__ void __launch_bounds__(256)
    k_keys_to_ids(unsigned long long *__restrict__ keys, long long n, int N, int K,
                  int32_t *__restrict__ ids, uint32_t *__restrict__ hist, int hist_tiles) {
  pdl_wait();
  for (long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x; r < n;
       r += (long long)gridDim.x * blockDim.x) {
    const unsigned long long key = keys[r];
    const int idx = (int)(0xFFFFFFFFu - (uint32_t)key);
    // every point gets a key from every chunk unless the assign gave up (its
    // timeout is in the device error word): then write 0 and count nothing
    const bool valid = key != 0ull && (unsigned)idx < (unsigned)K;
    ids[r] = valid ? idx : 0;
    if (hist && valid) {
      const long long b = r / N;
      const int row = (int)(r - b * N);
      atomicAdd(hist + ((size_t)b * hist_tiles + row / kSortTile) * K + idx, 1u);
    }
    keys[r] = 0ull;
  }
}

// ||x_i||^2 of every point, one thread per row, summed in exactly the order
// the norm warp uses on a shared tile (16-byte chunks in order; low halves into
// s0, high halves into s1; s0 + s1), so both give bit-identical norms and a
// Lloyd run that precomputes them assigns exactly like fk_assign.
template <typename T>
__global__ void __launch_bounds__(256)
    k_point_norms(const T *__restrict__ x, long long rows, int d, float *__restrict__ xn) {
  const int chunks = d / 8;
  for (long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x; r < rows;
       r += (long long)gridDim.x * blockDim.x) {
    const uint4 *row = reinterpret_cast<const uint4 *>(x + (size_t)r * d);
    float s0 = 0.f, s1 = 0.f;
    for (int j = 0; j < chunks; ++j) {
      const uint4 v = __ldg(row + j);
      sq2_acc<T>(v.x, s0, s1);
      sq2_acc<T>(v.y, s0, s1);
      sq2_acc<T>(v.z, s0, s1);
      sq2_acc<T>(v.w, s0, s1);
    }
    xn[r] = s0 + s1;
  }
}

template <typename T>
int point_norms_t(const void *x, long long rows, int d, float *xn, cudaStream_t s) {
  long long blocks = (rows + 255) / 256;
  const long long cap = (long long)num_sms() * 16;
  if (blocks > cap) blocks = cap;
  k_point_norms<T><<<(unsigned)blocks, 256, 0, s>>>(static_cast<const T *>(x), rows, d, xn);
  FK_TRY(launched());
  FK_CUDA(cudaGetLastError());
  return FK_OK;
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

// (inner, rows, B) tensor of dtype's elements (fp32 for FK_F32, else 16-bit),
// box (box_inner, box_rows, 1).
int encode_3d(CUtensorMap *map, const void *base, int dtype, int inner, long long rows, int B,
              int box_inner, int box_rows, CUtensorMapSwizzle swz) {
  EncodeTiledFn enc;
  FK_TRY(get_encoder(&enc));
  const cuuint64_t es = dtype == FK_F32 ? 4 : 2;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)B};
  cuuint64_t strides[2] = {(cuuint64_t)inner * es, (cuuint64_t)rows * inner * es};
  cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType ty = dtype == FK_F32    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : dtype == FK_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                    : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUresult r = enc(map, ty, 3, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(FK_ECUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)r));
  return FK_OK;
}

template <typename T, bool RESIDENT, int KB, int STAGES>
int launch_variant(const CUtensorMap &tmx, const CUtensorMap &tmc, const TcArgs &a, int grid, cudaStream_t s) {
  using L = Layout<RESIDENT, KB, STAGES>;
  FK_TRY(set_smem_limit((const void *)k_flash_assign<T, RESIDENT, KB, STAGES>, (int)L::kAlloc));
  FK_CUDA(launch_pdl(k_flash_assign<T, RESIDENT, KB, STAGES>, dim3(grid), dim3(kThreads), L::kAlloc, s, tmx, tmc,
                     a));
  FK_TRY(launched());
  FK_CUDA(cudaGetLastError());
  return FK_OK;
}

template <typename T>
int launch_typed(const CUtensorMap &tmx, const CUtensorMap &tmc, const TcArgs &a, int grid, cudaStream_t s) {
  // resident stages hold whole chunks: 4 x 40 KB (d <= 64) or 2 x 72 KB (d <= 128)
  if constexpr (sizeof(T) == 2) {
    if (a.kblocks == 1) return launch_variant<T, true, 1, 4>(tmx, tmc, a, grid, s);
    if (a.kblocks == 2) return launch_variant<T, true, 2, 2>(tmx, tmc, a, grid, s);
  }
  return launch_variant<T, false, 1, 4>(tmx, tmc, a, grid, s);
}

}  // namespace

int launch_point_norms(const void *x, int dtype, long long rows, int d, float *xn, cudaStream_t s) {
  if (dtype == FK_BF16) return point_norms_t<__nv_bfloat16>(x, rows, d, xn, s);
  return point_norms_t<__half>(x, rows, d, xn, s);
}

int launch_assign_tc(const void *x, const void *ch, const void *cnx, const float *xn, int dtype,
                     int B, long long N, int K, int d, long long Kpad, int32_t *ids, int *err,
                     cudaStream_t s, uint32_t *hist, unsigned long long *keys, float *xn_out) {
  // K-blocks are 128-byte rows: 64 16-bit elements or 32 fp32 (read as tf32);
  // norm rows are 32 bytes (16 or 8 elements), stored per 256-row chunk as
  // the shared-memory image of the swizzled tile and moved by bulk copies
  const int blk = dtype == FK_F32 ? 32 : kBlockK;
  if (Kpad != (long long)(K + kChunkN - 1) / kChunkN * kChunkN || (reinterpret_cast<uintptr_t>(cnx) & 15u))
    return set_error(FK_EINVAL, "extension rows: Kpad must be K rounded up to the chunk, 16-byte aligned");
  CUtensorMap tmx, tmc;
  FK_TRY(encode_3d(&tmx, x, dtype, d, N, B, blk, kTileM, CU_TENSOR_MAP_SWIZZLE_128B));
  FK_TRY(encode_3d(&tmc, ch, dtype, d, K, B, blk, kChunkN, CU_TENSOR_MAP_SWIZZLE_128B));
  TcArgs a;
  a.cnx = static_cast<const uint8_t *>(cnx);
  a.N = (int)N;
  a.K = K;
  a.hist = hist;
  a.hist_tiles = (int)((N + kSortTile - 1) / kSortTile);
  a.tiles_per_batch = (int)((N + kTileM - 1) / kTileM);
  long long total = (long long)B * a.tiles_per_batch;
  if (total > 0x7fffffffLL) return set_error(FK_EUNSUPPORTED, "too many point tiles");
  a.total_tiles = (int)total;
  a.nchunks = (K + kChunkN - 1) / kChunkN;
  a.kblocks = (d + blk - 1) / blk;
  a.xn = xn;
  a.xn_out = xn ? nullptr : xn_out;
  a.ids = ids;
  a.err = err;
  a.xg = x;
  a.cg = ch;
  a.d = d;
  a.idesc = sm100::idesc_f32acc(dtype == FK_F32 ? 2u : dtype == FK_BF16 ? 1u : 0u, kTileM, kChunkN);
  // split-d (fp32, or more than two 16-bit K-blocks): with keys, one work item
  // per (tile, chunk) and a merge of the chunks' results
  const bool splitd = dtype == FK_F32 || a.kblocks > 2;
  a.keys = (splitd && keys && total * a.nchunks <= 0x7fffffffLL) ? keys : nullptr;
  if (a.keys) a.hist = nullptr;  // counted when the ids are written
  const long long tasks = a.keys ? total * a.nchunks : total;
  int grid = num_sms();
  if (tasks < grid) grid = (int)tasks;
  if (dtype == FK_F32) FK_TRY(launch_typed<float>(tmx, tmc, a, grid, s));
  else if (dtype == FK_BF16) FK_TRY(launch_typed<__nv_bfloat16>(tmx, tmc, a, grid, s));
  else FK_TRY(launch_typed<__half>(tmx, tmc, a, grid, s));
  if (!a.keys) return FK_OK;
  const long long n = (long long)B * N;
  long long blocks = (n + 255) / 256;
  if (blocks > (long long)num_sms() * 8) blocks = (long long)num_sms() * 8;
  FK_CUDA(launch_pdl(k_keys_to_ids, dim3((unsigned)blocks), dim3(256), 0, s, keys, n, (int)N, K, ids, hist,
                     a.hist_tiles));
  FK_TRY(launched());
  return FK_OK;
}

}  // namespace fk
