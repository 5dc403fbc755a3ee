// Stable counting sort of the assignment vector (update steps a2-a4).
//
// The sort-inverse update orders the assignment vector by cluster id so that
// equal ids form contiguous segments, and keeps the inverse mapping (perm:
// sorted position -> point index) instead of moving the points
// ("Flash-KMeans: IO感知的精确K-Means", section "它攻克的兩大瓶頸", the
// paragraph on Sort-Inverse Update; "Flash-KMeans: Fast and Memory-Efficient
// Exact K-Means", Abstract).  The pages sort with an argsort; here it is a
// stable LSD counting sort by digits of at most 12 bits:
//   - one pass with the id itself as the digit when K <= 4096,
//   - two passes (low digit, then high digit) for larger K.
// Each pass has three kernels:
//   k_tile_hist    one warp per tile of 2048 points counts digits into its
//                  own shared-memory counters -> H[b][tile][bin],
//   k_scan         per batch: bin totals, a block scan over bins -> offsets,
//                  then the exclusive prefix over tiles of every bin, in place,
//   k_tile_scatter one warp per tile walks its points in order; equal digits
//                  inside a round of 32 are ranked with a per-bit ballot mask and
//                  the warp's cursor per bin starts at offsets[bin] + H[tile].
// Stability: tiles are ordered by the tile prefix, points inside a tile by the
// in-order rounds and the lane rank inside a round.
#include "fk_internal.h"

namespace fk {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr unsigned kNoDigit = 0xffffffffu;
constexpr int kTileWarps = 4;            // warps (= tiles) per CTA
constexpr int kRounds = kSortTile / 32;  // rounds of 32 points per tile

struct PassCfg {
  int shift;      // digit = (key >> shift) & mask
  unsigned mask;  // a single pass with bins = K keeps the whole id
  int bins;
  int nbits;      // bits needed for a digit (ceil(log2(bins)))
  bool check;     // validate 0 <= key < K (first pass over caller ids)
};

// Lanes of the warp holding the same digit as this lane, from one ballot per
// digit bit (invalid lanes, digit kNoDigit, match nobody).  Cheaper than a
// general match instruction for digits of at most 12 bits.
__device__ __forceinline__ unsigned peers_of(unsigned dg, int nbits) {
  const bool valid = dg != 0xffffffffu;
  unsigned peers = __ballot_sync(0xffffffffu, valid);
  for (int bit = 0; bit < nbits; ++bit) {
    const bool on = (dg >> bit) & 1u;
    const unsigned bal = __ballot_sync(0xffffffffu, on);
    peers &= on ? bal : ~bal;
  }
  return valid ? peers : 0u;
}

__device__ __forceinline__ unsigned digit_of(int key, bool valid, const PassCfg &pc, int K,
                                             int *err) {
  if (!valid) return kNoDigit;
  if (pc.check && (key < 0 || key >= K)) {
    atomicCAS(err, DEV_OK, DEV_BAD_ID);
    return kNoDigit;
  }
  return ((unsigned)key >> pc.shift) & pc.mask;
}

// Copies the tile's values (fewer at the end of a batch) into this warp's shared
// buffer with asynchronous 4-byte copies (no register round trip, all in
// flight at once), then waits for them.  Positions past n are zero-filled.
__device__ __forceinline__ void stage_tile(int32_t *dst, const int32_t *src, long long base,
                                           long long n, int lane) {
#pragma unroll 8
  for (int r = 0; r < kRounds; ++r) {
    const long long i = base + r * 32 + lane;
    const bool in = i < n;
    const int32_t *p = src + (in ? i : 0);
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst + r * 32 + lane));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(d), "l"(p), "r"(in ? 4 : 0)
                 : "memory");
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncwarp();
}

// H[b][tile][bin] = number of points of this tile with this digit.
__global__ void __launch_bounds__(kTileWarps * 32) k_tile_hist(const int32_t *__restrict__ keys,
                                                                int N, int K, int T, PassCfg pc,
                                                                uint32_t *__restrict__ H, int *err) {
  extern __shared__ uint32_t cnt_all[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x * kTileWarps + warp;
  const int b = blockIdx.y;
  if (tile >= T) return;
  const int bins = pc.bins;
  uint32_t *cnt = cnt_all + warp * (bins + kSortTile);
  int32_t *sk = reinterpret_cast<int32_t *>(cnt + bins);
  const int32_t *kb = keys + (size_t)b * N;
  const long long base = (long long)tile * kSortTile;
  stage_tile(sk, kb, base, N, lane);
  for (int e = lane; e < bins; e += 32) cnt[e] = 0;
  __syncwarp();
  for (int r = 0; r < kRounds; ++r) {
    const long long i = base + r * 32 + lane;
    const bool valid = i < N;
    const int key = sk[r * 32 + lane];
    const unsigned dg = digit_of(key, valid, pc, K, err);
    const unsigned peers = peers_of(dg, pc.nbits);
    if (dg != kNoDigit && lane == __ffs(peers) - 1) cnt[dg] += __popc(peers);
    __syncwarp();
  }
  uint32_t *hb = H + ((size_t)b * T + tile) * bins;
  for (int e = lane; e < bins; e += 32) hb[e] = cnt[e];
}

// One CTA per batch over H[b][T][bins]:
//   offsets[b][bin] = sum of the totals of earlier bins,
//   counts[b][bin]  = total of the bin (optional; accumulate adds to it),
//   H[b][t][bin]    = sum over tiles t' < t of the bin (in place).
__global__ void __launch_bounds__(1024) k_scan(uint32_t *__restrict__ H, int bins, int T,
                                               int32_t *__restrict__ counts,
                                               int32_t *__restrict__ offsets, int accumulate) {
  __shared__ uint32_t wsum[32];
  const int b = blockIdx.x;
  uint32_t *hb = H + (size_t)b * T * bins;
  const int per = (bins + (int)blockDim.x - 1) / (int)blockDim.x;
  const int lo = min(bins, (int)threadIdx.x * per), hi = min(bins, lo + per);
  uint32_t local = 0;
  for (int bin = lo; bin < hi; ++bin)
    for (int t = 0; t < T; ++t) local += hb[(size_t)t * bins + bin];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t v = lane < (int)(blockDim.x >> 5) ? wsum[lane] : 0;
    uint32_t vi = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(kFull, vi, o);
      if (lane >= o) vi += u;
    }
    wsum[lane] = vi - v;
  }
  __syncthreads();
  uint32_t run = wsum[warp] + incl - local;
  for (int bin = lo; bin < hi; ++bin) {
    if (offsets) offsets[(size_t)b * bins + bin] = (int32_t)run;
    uint32_t t_run = 0;
    for (int t = 0; t < T; ++t) {
      const uint32_t v = hb[(size_t)t * bins + bin];
      hb[(size_t)t * bins + bin] = t_run;
      t_run += v;
    }
    if (counts) {
      int32_t *dst = counts + (size_t)b * bins + bin;
      *dst = accumulate ? *dst + (int32_t)t_run : (int32_t)t_run;
    }
    run += t_run;
  }
}

// Stable scatter: vals_out[pos] = vals_in ? vals_in[i] : i and keys_out[pos] = key,
// pos = offsets[digit] + H[tile][digit] + rank of the point among the tile's
// earlier points with the same digit.
__global__ void __launch_bounds__(kTileWarps * 32) k_tile_scatter(
    const int32_t *__restrict__ keys, const int32_t *__restrict__ vals_in, int N, int K, int T,
    PassCfg pc, const uint32_t *__restrict__ G, const int32_t *__restrict__ offsets,
    int32_t *__restrict__ keys_out, int32_t *__restrict__ vals_out, int *err) {
  extern __shared__ uint32_t cur_all[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x * kTileWarps + warp;
  const int b = blockIdx.y;
  if (tile >= T) return;
  const int bins = pc.bins;
  uint32_t *cur = cur_all + warp * (bins + 2 * kSortTile);
  int32_t *sk = reinterpret_cast<int32_t *>(cur + bins);
  int32_t *sv = sk + kSortTile;
  const int32_t *kb = keys + (size_t)b * N;
  int32_t *ko = keys_out ? keys_out + (size_t)b * N : nullptr;
  int32_t *vo = vals_out + (size_t)b * N;
  const int32_t *vi = vals_in ? vals_in + (size_t)b * N : nullptr;
  const long long base = (long long)tile * kSortTile;
  stage_tile(sk, kb, base, N, lane);
  if (vi) stage_tile(sv, vi, base, N, lane);
  const uint32_t *gb = G + ((size_t)b * T + tile) * bins;
  const int32_t *ob = offsets + (size_t)b * bins;
  for (int e = lane; e < bins; e += 32) cur[e] = gb[e] + (uint32_t)ob[e];
  __syncwarp();
  const unsigned lt = (1u << lane) - 1u;
  for (int r = 0; r < kRounds; ++r) {
    const long long i = base + r * 32 + lane;
    const bool valid = i < N;
    const int key = sk[r * 32 + lane];
    const unsigned dg = digit_of(key, valid, pc, K, err);
    const unsigned peers = peers_of(dg, pc.nbits);
    uint32_t pos = 0;
    if (dg != kNoDigit) pos = cur[dg] + __popc(peers & lt);
    __syncwarp();
    if (dg != kNoDigit) {
      if (lane == __ffs(peers) - 1) cur[dg] += __popc(peers);
      vo[pos] = vi ? sv[r * 32 + lane] : (int32_t)i;
      if (ko) ko[pos] = key;
    }
    __syncwarp();
  }
}

// counts[b][k] += #{i : keys[b][i] = k} (counts for K too large for one pass).
__global__ void __launch_bounds__(256) k_count(const int32_t *__restrict__ keys, int N, int K,
                                               int32_t *__restrict__ counts, int use_smem) {
  extern __shared__ int32_t hs[];
  const int b = blockIdx.y;
  if (use_smem) {
    for (int e = threadIdx.x; e < K; e += blockDim.x) hs[e] = 0;
    __syncthreads();
  }
  const int32_t *kb = keys + (size_t)b * N;
  const long long i0 = (long long)blockIdx.x * kSortTile;
  for (long long i = i0 + threadIdx.x; i < i0 + kSortTile && i < N; i += blockDim.x) {
    const int k = kb[i];
    if (k < 0 || k >= K) continue;
    if (use_smem) atomicAdd(&hs[k], 1);
    else atomicAdd(&counts[(size_t)b * K + k], 1);
  }
  if (use_smem) {
    __syncthreads();
    for (int e = threadIdx.x; e < K; e += blockDim.x)
      if (hs[e]) atomicAdd(&counts[(size_t)b * K + e], hs[e]);
  }
}

int bits_for(int K) {
  int n = 0;
  while (n < 31 && (1LL << n) < (long long)K) ++n;
  return n;
}

int set_attrs() {
  static bool done = false;
  if (done) return FK_OK;
  const int hist_max = kTileWarps * ((1 << kMaxDigitBits) + kSortTile) * 4;
  const int scat_max = kTileWarps * ((1 << kMaxDigitBits) + 2 * kSortTile) * 4;
  FK_CUDA(cudaFuncSetAttribute(k_tile_hist, cudaFuncAttributeMaxDynamicSharedMemorySize, hist_max));
  FK_CUDA(cudaFuncSetAttribute(k_tile_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize, scat_max));
  FK_CUDA(cudaFuncSetAttribute(k_count, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024));
  done = true;
  return FK_OK;
}

int one_pass(Workspace *ws, const int32_t *keys_in, const int32_t *vals_in, int B, int N, int K,
             int T, PassCfg pc, int32_t *counts, int32_t *offsets, bool accumulate,
             int32_t *keys_out, int32_t *vals_out, cudaStream_t s) {
  FK_TRY(ensure(ws->table, (size_t)B * T * pc.bins * sizeof(uint32_t)));
  uint32_t *H = (uint32_t *)ws->table.p;
  dim3 grid((unsigned)((T + kTileWarps - 1) / kTileWarps), (unsigned)B);
  const size_t shm_h = (size_t)kTileWarps * (pc.bins + kSortTile) * sizeof(uint32_t);
  const size_t shm_s = (size_t)kTileWarps * (pc.bins + 2 * kSortTile) * sizeof(uint32_t);
  k_tile_hist<<<grid, kTileWarps * 32, shm_h, s>>>(keys_in, N, K, T, pc, H, ws->err);
  count_launch();
  FK_CUDA(cudaGetLastError());
  k_scan<<<B, 1024, 0, s>>>(H, pc.bins, T, counts, offsets, accumulate ? 1 : 0);
  count_launch();
  FK_CUDA(cudaGetLastError());
  k_tile_scatter<<<grid, kTileWarps * 32, shm_s, s>>>(keys_in, vals_in, N, K, T, pc, H, offsets,
                                                    keys_out, vals_out, ws->err);
  count_launch();
  FK_CUDA(cudaGetLastError());
  return FK_OK;
}

}  // namespace

int run_sort(Workspace *ws, const int32_t *ids, int B, long long N_, int K, int32_t *counts,
             int32_t *offsets, int32_t *perm, int32_t *keys_out, cudaStream_t s) {
  FK_TRY(set_attrs());
  const int N = (int)N_;
  const int T = (int)((N_ + kSortTile - 1) / kSortTile);
  const int nbits = bits_for(K);
  if (nbits <= kMaxDigitBits) {
    int32_t *off = offsets;
    if (!off) {
      FK_TRY(ensure(ws->offsets, (size_t)B * K * sizeof(int32_t)));
      off = (int32_t *)ws->offsets.p;
    }
    PassCfg pc{0, 0xffffffffu, K, nbits, true};
    return one_pass(ws, ids, nullptr, B, N, K, T, pc, counts, off, false, keys_out, perm, s);
  }
  const int lo = (nbits + 1) / 2, hi = nbits - lo;
  const size_t nb = (size_t)B * N * sizeof(int32_t);
  FK_TRY(ensure(ws->keys_b, nb));
  FK_TRY(ensure(ws->vals_b, nb));
  int32_t *kt = (int32_t *)ws->keys_b.p, *vt = (int32_t *)ws->vals_b.p;
  // digit offsets of the passes live in the workspace (at most 4096 per batch)
  FK_TRY(ensure(ws->digit_off, (size_t)B * (1 << kMaxDigitBits) * sizeof(int32_t)));
  int32_t *doff = (int32_t *)ws->digit_off.p;
  PassCfg p1{0, (1u << lo) - 1u, 1 << lo, lo, true};
  FK_TRY(one_pass(ws, ids, nullptr, B, N, K, T, p1, nullptr, doff, false, kt, vt, s));
  PassCfg p2{lo, (1u << hi) - 1u, 1 << hi, hi, false};
  FK_TRY(one_pass(ws, kt, vt, B, N, K, T, p2, nullptr, doff, false, keys_out, perm, s));
  if (counts || offsets) {
    int32_t *cnt = counts;
    if (!cnt) {
      FK_TRY(ensure(ws->counts, (size_t)B * K * sizeof(int32_t)));
      cnt = (int32_t *)ws->counts.p;
    }
    FK_CUDA(cudaMemsetAsync(cnt, 0, (size_t)B * K * sizeof(int32_t), s));
    const int use_smem = (size_t)K * 4 <= 64 * 1024 ? 1 : 0;
    dim3 grid((unsigned)T, (unsigned)B);
    k_count<<<grid, 256, use_smem ? K * 4 : 0, s>>>(ids, N, K, cnt, use_smem);
    count_launch();
    FK_CUDA(cudaGetLastError());
    if (offsets) {
      // offsets = exclusive scan of the counts (a table with one tile)
      FK_TRY(ensure(ws->table, (size_t)B * K * sizeof(uint32_t)));
      FK_CUDA(cudaMemcpyAsync(ws->table.p, cnt, (size_t)B * K * sizeof(int32_t),
                              cudaMemcpyDeviceToDevice, s));
      k_scan<<<B, 1024, 0, s>>>((uint32_t *)ws->table.p, K, 1, nullptr, offsets, 0);
      count_launch();
      FK_CUDA(cudaGetLastError());
    }
  }
  return FK_OK;
}

}  // namespace fk
