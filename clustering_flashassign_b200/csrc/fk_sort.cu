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
// Each pass is: per-tile histograms (4096 points per CTA, per-warp counters in
// shared memory) -> one exclusive scan per batch over the bin-major
// (bin, tile) table -> a stable scatter in which every warp walks its points
// in order and ranks equal digits with __match_any_sync.  Stability follows
// from the bin-major scan (earlier tiles first), the warp-major base inside a
// tile and the in-order rounds inside a warp.
#include "fk_internal.h"

namespace fk {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr unsigned kNoDigit = 0xffffffffu;

struct PassCfg {
  int shift;      // digit = (key >> shift) & mask
  unsigned mask;  // for a single pass with bins = K the mask keeps the whole id
  int bins;
  bool check;     // validate 0 <= key < K (first pass over caller ids)
};

__device__ __forceinline__ unsigned digit_of(int key, bool valid, const PassCfg &pc, int K,
                                             int *err) {
  if (!valid) return kNoDigit;
  if (pc.check && (key < 0 || key >= K)) {
    atomicCAS(err, DEV_OK, DEV_BAD_ID);
    return kNoDigit;
  }
  return ((unsigned)key >> pc.shift) & pc.mask;
}

// H[b][bin][tile] = number of points of this tile with this digit.
__global__ void __launch_bounds__(kSortWarps * 32) k_tile_hist(const int32_t *__restrict__ keys,
                                                                int N, int K, int T, PassCfg pc,
                                                                uint32_t *__restrict__ H, int *err) {
  extern __shared__ uint16_t hist16[];  // [kSortWarps][bins]
  const int tile = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bins = pc.bins;
  for (int e = threadIdx.x; e < kSortWarps * bins; e += blockDim.x) hist16[e] = 0;
  __syncthreads();
  const int32_t *kb = keys + (size_t)b * N;
  uint16_t *mine = hist16 + warp * bins;
  const long long base = (long long)tile * kSortTile + warp * (kSortRounds * 32);
  for (int r = 0; r < kSortRounds; ++r) {
    long long i = base + r * 32 + lane;
    bool valid = i < N;
    int key = valid ? kb[i] : 0;
    unsigned dg = digit_of(key, valid, pc, K, err);
    unsigned peers = __match_any_sync(kFull, dg);
    if (dg != kNoDigit && lane == __ffs(peers) - 1) mine[dg] += (uint16_t)__popc(peers);
    __syncwarp();
  }
  __syncthreads();
  uint32_t *hb = H + (size_t)b * bins * T;
  for (int bin = threadIdx.x; bin < bins; bin += blockDim.x) {
    uint32_t s = 0;
#pragma unroll
    for (int w = 0; w < kSortWarps; ++w) s += hist16[w * bins + bin];
    hb[(size_t)bin * T + tile] = s;
  }
}

// Per batch: counts (sum over tiles, optional), exclusive scan of the
// bin-major table in place, offsets = scanned value of tile 0 (optional).
__global__ void __launch_bounds__(1024) k_scan(uint32_t *__restrict__ H, int bins, int T,
                                               int32_t *__restrict__ counts,
                                               int32_t *__restrict__ offsets, int accumulate) {
  __shared__ uint32_t wsum[32];
  const int b = blockIdx.x;
  uint32_t *hb = H + (size_t)b * bins * T;
  if (counts) {
    for (int bin = threadIdx.x; bin < bins; bin += blockDim.x) {
      uint32_t s = 0;
      for (int t = 0; t < T; ++t) s += hb[(size_t)bin * T + t];
      int32_t *dst = counts + (size_t)b * bins + bin;
      *dst = accumulate ? *dst + (int32_t)s : (int32_t)s;
    }
    __syncthreads();
  }
  const long long M = (long long)bins * T;
  const long long L = (M + blockDim.x - 1) / blockDim.x;
  const long long lo = threadIdx.x * L, hi = lo + L < M ? lo + L : M;
  uint32_t local = 0;
  for (long long e = lo; e < hi; ++e) local += hb[e];
  // block exclusive scan of `local`
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t v = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t v = lane < (int)(blockDim.x >> 5) ? wsum[lane] : 0;
    uint32_t vi = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t u = __shfl_up_sync(kFull, vi, o);
      if (lane >= o) vi += u;
    }
    wsum[lane] = vi - v;  // exclusive
  }
  __syncthreads();
  uint32_t run = wsum[warp] + incl - local;
  for (long long e = lo; e < hi; ++e) {
    uint32_t v = hb[e];
    hb[e] = run;
    run += v;
  }
  if (offsets) {
    __syncthreads();
    for (int bin = threadIdx.x; bin < bins; bin += blockDim.x)
      offsets[(size_t)b * bins + bin] = (int32_t)hb[(size_t)bin * T];
  }
}

// Stable scatter: vals_out[pos] = vals_in ? vals_in[i] : i, keys_out[pos] = key.
__global__ void __launch_bounds__(kSortWarps * 32) k_tile_scatter(
    const int32_t *__restrict__ keys, const int32_t *__restrict__ vals_in, int N, int K, int T,
    PassCfg pc, const uint32_t *__restrict__ G, int32_t *__restrict__ keys_out,
    int32_t *__restrict__ vals_out, int *err) {
  extern __shared__ uint32_t cur[];  // [kSortWarps][bins]
  const int tile = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bins = pc.bins;
  for (int e = threadIdx.x; e < kSortWarps * bins; e += blockDim.x) cur[e] = 0;
  __syncthreads();
  const int32_t *kb = keys + (size_t)b * N;
  uint32_t *mine = cur + warp * bins;
  const long long base = (long long)tile * kSortTile + warp * (kSortRounds * 32);
  // 1) per-warp counts
  for (int r = 0; r < kSortRounds; ++r) {
    long long i = base + r * 32 + lane;
    bool valid = i < N;
    int key = valid ? kb[i] : 0;
    unsigned dg = digit_of(key, valid, pc, K, err);
    unsigned peers = __match_any_sync(kFull, dg);
    if (dg != kNoDigit && lane == __ffs(peers) - 1) mine[dg] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // 2) warp-major exclusive bases on top of the tile's global base
  const uint32_t *gb = G + (size_t)b * bins * T;
  for (int bin = threadIdx.x; bin < bins; bin += blockDim.x) {
    uint32_t run = gb[(size_t)bin * T + tile];
#pragma unroll
    for (int w = 0; w < kSortWarps; ++w) {
      uint32_t c = cur[w * bins + bin];
      cur[w * bins + bin] = run;
      run += c;
    }
  }
  __syncthreads();
  // 3) in-order rounds: rank among equal digits, write, advance the cursor
  int32_t *ko = keys_out ? keys_out + (size_t)b * N : nullptr;
  int32_t *vo = vals_out + (size_t)b * N;
  const int32_t *vi = vals_in ? vals_in + (size_t)b * N : nullptr;
  const unsigned lt = (1u << lane) - 1u;
  for (int r = 0; r < kSortRounds; ++r) {
    long long i = base + r * 32 + lane;
    bool valid = i < N;
    int key = valid ? kb[i] : 0;
    unsigned dg = digit_of(key, valid, pc, K, err);
    unsigned peers = __match_any_sync(kFull, dg);
    uint32_t pos = 0;
    if (dg != kNoDigit) pos = mine[dg] + __popc(peers & lt);
    __syncwarp();
    if (dg != kNoDigit) {
      if (lane == __ffs(peers) - 1) mine[dg] += __popc(peers);
      vo[pos] = vi ? vi[i] : (int32_t)i;
      if (ko) ko[pos] = key;
    }
    __syncwarp();
  }
}

// counts[b][k] (+)= #{i : keys[b][i] = k}, for K too large for a single pass.
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
    int k = kb[i];
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

bool g_attr_done = false;

int set_attrs() {
  if (g_attr_done) return FK_OK;
  FK_CUDA(cudaFuncSetAttribute(k_tile_hist, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kSortWarps * (1 << kMaxDigitBits) * 2));
  FK_CUDA(cudaFuncSetAttribute(k_tile_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kSortWarps * (1 << kMaxDigitBits) * 4));
  FK_CUDA(cudaFuncSetAttribute(k_count, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024));
  g_attr_done = true;
  return FK_OK;
}

int one_pass(Workspace *ws, const int32_t *keys_in, const int32_t *vals_in, int B, int N, int K,
             int T, PassCfg pc, int32_t *counts, int32_t *offsets, bool accumulate,
             int32_t *keys_out, int32_t *vals_out, cudaStream_t s) {
  size_t tbytes = (size_t)B * pc.bins * T * sizeof(uint32_t);
  FK_TRY(ensure(ws->table, tbytes));
  uint32_t *H = (uint32_t *)ws->table.p;
  dim3 grid((unsigned)T, (unsigned)B);
  k_tile_hist<<<grid, kSortWarps * 32, kSortWarps * pc.bins * 2, s>>>(keys_in, N, K, T, pc, H, ws->err);
  count_launch();
  FK_CUDA(cudaGetLastError());
  k_scan<<<B, 1024, 0, s>>>(H, pc.bins, T, counts, offsets, accumulate ? 1 : 0);
  count_launch();
  FK_CUDA(cudaGetLastError());
  k_tile_scatter<<<grid, kSortWarps * 32, kSortWarps * pc.bins * 4, s>>>(keys_in, vals_in, N, K, T, pc, H, keys_out, vals_out, ws->err);
  count_launch();
  FK_CUDA(cudaGetLastError());
  return FK_OK;
}

}  // namespace

int run_sort(Workspace *ws, const int32_t *ids, int B, long long N_, int K, int32_t *counts,
             int32_t *offsets, int32_t *perm, int32_t *keys_out, bool accumulate_counts,
             cudaStream_t s) {
  FK_TRY(set_attrs());
  const int N = (int)N_;
  const int T = (int)((N_ + kSortTile - 1) / kSortTile);
  const int nbits = bits_for(K);
  if (nbits <= kMaxDigitBits) {
    PassCfg pc{0, 0xffffffffu, K, true};
    return one_pass(ws, ids, nullptr, B, N, K, T, pc, counts, offsets, accumulate_counts,
                    keys_out, perm, s);
  }
  const int lo = (nbits + 1) / 2, hi = nbits - lo;
  size_t nb = (size_t)B * N * sizeof(int32_t);
  FK_TRY(ensure(ws->keys_b, nb));
  FK_TRY(ensure(ws->vals_b, nb));
  int32_t *kt = (int32_t *)ws->keys_b.p, *vt = (int32_t *)ws->vals_b.p;
  PassCfg p1{0, (1u << lo) - 1u, 1 << lo, true};
  FK_TRY(one_pass(ws, ids, nullptr, B, N, K, T, p1, nullptr, nullptr, false, kt, vt, s));
  PassCfg p2{lo, (1u << hi) - 1u, 1 << hi, false};
  FK_TRY(one_pass(ws, kt, vt, B, N, K, T, p2, nullptr, nullptr, false, keys_out, perm, s));
  if (counts || offsets) {
    int32_t *cnt = counts;
    if (!cnt) {
      FK_TRY(ensure(ws->counts, (size_t)B * K * sizeof(int32_t)));
      cnt = (int32_t *)ws->counts.p;
    }
    if (!accumulate_counts || cnt != counts) FK_CUDA(cudaMemsetAsync(cnt, 0, (size_t)B * K * sizeof(int32_t), s));
    int use_smem = (size_t)K * 4 <= 64 * 1024 ? 1 : 0;
    dim3 grid((unsigned)T, (unsigned)B);
    k_count<<<grid, 256, use_smem ? K * 4 : 0, s>>>(ids, N, K, cnt, use_smem);
    count_launch();
    FK_CUDA(cudaGetLastError());
    if (offsets) {
      FK_CUDA(cudaMemcpyAsync(offsets, cnt, (size_t)B * K * sizeof(int32_t), cudaMemcpyDeviceToDevice, s));
      k_scan<<<B, 1024, 0, s>>>((uint32_t *)offsets, K, 1, nullptr, nullptr, 0);
      count_launch();
      FK_CUDA(cudaGetLastError());
    }
  }
  return FK_OK;
}

}  // namespace fk
