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
// Each pass has three kernels over tiles of 2048 points (one CTA of 8 warps
// per tile; warp w owns the tile's points 256w .. 256w+255, 8 rounds of 32):
//   k_tile_hist    each warp counts its digits into its own shared counters;
//                  the CTA sums the 8 warps -> H[b][tile][bin],
//   k_scan_tiles   per (32 bins, batch): the exclusive prefix over tiles of
//                  every bin, in place, and the bin totals -> counts,
//   k_tile_scatter block scan of the counts -> bin offsets (written once per
//                  batch) plus H[tile][bin] -> the tile's bases; per-warp
//                  counts again, their prefix over the 8 warps on top of the
//                  bases, then every warp ranks its rounds in order: equal
//                  digits inside a round are ranked with a per-bit ballot
//                  mask.  The update takes the sorted (id, point) pairs as one
//                  8-byte store per point.
// Stability: tiles are ordered by the tile prefix, warps inside a tile by the
// warp prefix, points of a warp by the in-order rounds and the lane rank.
#include "fk_internal.h"

namespace fk {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr unsigned kNoDigit = 0xffffffffu;
constexpr int kSortWarps = 8;                          // warps per tile (CTA)
constexpr int kWarpPoints = kSortTile / kSortWarps;    // 256 points per warp
constexpr int kRounds = kWarpPoints / 32;              // rounds of 32 points per warp
constexpr int kSortThreads = kSortWarps * 32;

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
  const bool valid = dg != kNoDigit;
  unsigned peers = __ballot_sync(kFull, valid);
  for (int bit = 0; bit < nbits; ++bit) {
    const bool on = (dg >> bit) & 1u;
    const unsigned bal = __ballot_sync(kFull, on);
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

// This warp's keys (kRounds per lane, round r = points 32r..32r+31 of the
// warp's range), their digits and per-round peer masks.
struct WarpKeys {
  int key[kRounds];
  unsigned dg[kRounds];
  unsigned peers[kRounds];
};

__device__ __forceinline__ void fetch_warp_keys(WarpKeys &wk, const int32_t *kb, long long base,
                                                int N, int lane) {
#pragma unroll
  for (int r = 0; r < kRounds; ++r) {
    const long long i = base + r * 32 + lane;
    wk.key[r] = i < N ? __ldg(kb + i) : 0;
  }
}

__device__ __forceinline__ void rank_warp_keys(WarpKeys &wk, long long base, int N,
                                               const PassCfg &pc, int K, int *err, int lane) {
#pragma unroll
  for (int r = 0; r < kRounds; ++r) {
    const long long i = base + r * 32 + lane;
    wk.dg[r] = digit_of(wk.key[r], i < N, pc, K, err);
    wk.peers[r] = peers_of(wk.dg[r], pc.nbits);
  }
}

__device__ __forceinline__ void load_warp_keys(WarpKeys &wk, const int32_t *kb, long long base,
                                               int N, const PassCfg &pc, int K, int *err,
                                               int lane) {
  fetch_warp_keys(wk, kb, base, N, lane);
  rank_warp_keys(wk, base, N, pc, K, err, lane);
}

// cnt[dg] += number of this warp's points with digit dg (one leader per round
// and digit; the warp owns cnt).
__device__ __forceinline__ void count_warp(uint32_t *cnt, const WarpKeys &wk, int lane) {
#pragma unroll
  for (int r = 0; r < kRounds; ++r) {
    const unsigned dg = wk.dg[r], peers = wk.peers[r];
    if (dg != kNoDigit && lane == __ffs(peers) - 1) cnt[dg] += __popc(peers);
    __syncwarp();
  }
}

// out[bin] = gb[bin] + sum of counts[bin'] over bin' < bin, for bins <=
// kSortThreads * 16: the first sorted position of the tile's points with this
// digit (a block-wide exclusive scan; every thread of the CTA calls it).  The
// counts and the tile prefixes gb are fetched in one pass, so their latencies
// overlap.
__device__ __forceinline__ void tile_bases(const int32_t *counts, const uint32_t *gb, int bins,
                                           uint32_t *out) {
  __shared__ uint32_t wsum[kSortWarps];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int per = (bins + kSortThreads - 1) / kSortThreads;
  const int lo = min(bins, t * per), hi = min(bins, lo + per);
  uint32_t local = 0;
  for (int bin = lo; bin < hi; ++bin) {
    local += (uint32_t)__ldg(counts + bin);
    out[bin] = gb[bin];  // a plain load: the scatter may zero this row afterwards
  }
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t v = lane < kSortWarps ? wsum[lane] : 0;
    uint32_t vi = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(kFull, vi, o);
      if (lane >= o) vi += u;
    }
    if (lane < kSortWarps) wsum[lane] = vi - v;
  }
  __syncthreads();
  uint32_t run = wsum[warp] + incl - local;
  for (int bin = lo; bin < hi; ++bin) {
    out[bin] += run;
    run += (uint32_t)__ldg(counts + bin);
  }
  __syncthreads();
}

// H[b][tile][bin] = number of points of this tile with this digit.
__global__ void __launch_bounds__(kSortThreads) k_tile_hist(const int32_t *__restrict__ keys, int N,
                                                            int K, int T, PassCfg pc,
                                                            uint32_t *__restrict__ H, int *err) {
  extern __shared__ uint32_t cnt_all[];  // [kSortWarps][bins]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, b = blockIdx.y;
  const int bins = pc.bins;
  for (int e = threadIdx.x; e < kSortWarps * bins; e += kSortThreads) cnt_all[e] = 0;
  WarpKeys wk;
  load_warp_keys(wk, keys + (size_t)b * N, (long long)tile * kSortTile + warp * kWarpPoints, N, pc,
                 K, err, lane);
  __syncthreads();
  count_warp(cnt_all + warp * bins, wk, lane);
  __syncthreads();
  uint32_t *hb = H + ((size_t)b * T + tile) * bins;
  for (int bin = threadIdx.x; bin < bins; bin += kSortThreads) {
    uint32_t t = 0;
#pragma unroll
    for (int w = 0; w < kSortWarps; ++w) t += cnt_all[w * bins + bin];
    hb[bin] = t;
  }
}

// Grid (ceil(bins / 32), B): lane = bin, warp w = a contiguous range of tiles.
//   H[b][t][bin] <- sum over tiles t' < t of the bin (in place),
//   counts[b][bin] = the bin's total.
__global__ void __launch_bounds__(kSortThreads) k_scan_tiles(uint32_t *__restrict__ H, int bins,
                                                             int T, int32_t *__restrict__ counts,
                                                             unsigned *__restrict__ zero_word) {
  __shared__ uint32_t part[kSortWarps][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  // the update's max-shift word, zeroed here rather than by a memset that
  // would break the chain of dependent launches
  if (zero_word && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *zero_word = 0u;
  const int b = blockIdx.y, bin = blockIdx.x * 32 + lane;
  const bool on = bin < bins;
  const int per = (T + kSortWarps - 1) / kSortWarps;
  const int t0 = min(T, warp * per), t1 = min(T, t0 + per);
  uint32_t *hb = H + (size_t)b * T * bins + bin;
  uint32_t local = 0;
  if (on)
    for (int t = t0; t < t1; ++t) local += hb[(size_t)t * bins];
  part[warp][lane] = local;
  __syncthreads();
  if (warp == 0) {
    uint32_t run = 0;
#pragma unroll
    for (int w = 0; w < kSortWarps; ++w) {
      const uint32_t v = part[w][lane];
      part[w][lane] = run;
      run += v;
    }
    if (on) counts[(size_t)b * bins + bin] = (int32_t)run;
  }
  __syncthreads();
  if (on) {
    uint32_t run = part[warp][lane];
    for (int t = t0; t < t1; ++t) {
      const uint32_t v = hb[(size_t)t * bins];
      hb[(size_t)t * bins] = run;
      run += v;
    }
  }
}

// Stable scatter of tile `tile`: the point at position i goes to
// pos = offsets[digit] + G[tile][digit] + (earlier warps of the tile with the
// digit) + rank of the point among the warp's earlier points with the digit.
// It writes vals_out[pos] = vals_in ? vals_in[i] : i and keys_out[pos] = key
// (each when not NULL), or the pair kv_out[pos] = (key, value): one 8-byte
// store per point where the update needs both.  The CTA of tile 0 also writes
// offsets_out[b] (when not NULL) and -1 entries past the counted points (when
// an id was out of range).  zero_g: the tile's row of G is zeroed once
// read, so a histogram that the assign accumulates starts from zero again.
__global__ void __launch_bounds__(kSortThreads) k_tile_scatter(
    const int32_t *__restrict__ keys, const int32_t *__restrict__ vals_in, int N, int K, int T,
    PassCfg pc, uint32_t *__restrict__ G, const int32_t *__restrict__ counts,
    int32_t *__restrict__ offsets_out, int32_t *__restrict__ keys_out,
    int32_t *__restrict__ vals_out, int2 *__restrict__ kv_out, int zero_g, int *err) {
  extern __shared__ uint32_t sm[];  // base[bins], cnt[kSortWarps][bins]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, b = blockIdx.y;
  const int bins = pc.bins;
  uint32_t *tb = sm;
  uint32_t *cnt_all = sm + bins;
  const long long base = (long long)tile * kSortTile + warp * kWarpPoints;
  for (int e = threadIdx.x; e < kSortWarps * bins; e += kSortThreads) cnt_all[e] = 0;
  pdl_wait();
  pdl_trigger();
  // the keys (and values) are fetched first; their latency overlaps the scan
  WarpKeys wk;
  fetch_warp_keys(wk, keys + (size_t)b * N, base, N, lane);
  int vals[kRounds];
  if (vals_in) {
#pragma unroll
    for (int r = 0; r < kRounds; ++r) {
      const long long i = base + r * 32 + lane;
      vals[r] = i < N ? __ldg(vals_in + (size_t)b * N + i) : 0;
    }
  }
  uint32_t *grow = G + ((size_t)b * T + tile) * bins;
  tile_bases(counts + (size_t)b * bins, grow, bins, tb);  // ends with __syncthreads
  if (zero_g)
    for (int bin = threadIdx.x; bin < bins; bin += kSortThreads) grow[bin] = 0u;
  if (tile == 0 && offsets_out)  // tile 0's prefix is zero: its bases are the offsets
    for (int bin = threadIdx.x; bin < bins; bin += kSortThreads)
      offsets_out[(size_t)b * bins + bin] = (int32_t)tb[bin];
  rank_warp_keys(wk, base, N, pc, K, err, lane);
  uint32_t *cnt = cnt_all + warp * bins;
  count_warp(cnt, wk, lane);
  __syncthreads();
  for (int bin = threadIdx.x; bin < bins; bin += kSortThreads) {
    uint32_t run = tb[bin];
#pragma unroll
    for (int w = 0; w < kSortWarps; ++w) {
      const uint32_t v = cnt_all[w * bins + bin];
      cnt_all[w * bins + bin] = run;
      run += v;
    }
  }
  __syncthreads();
  int32_t *ko = keys_out ? keys_out + (size_t)b * N : nullptr;
  int32_t *vo = vals_out ? vals_out + (size_t)b * N : nullptr;
  int2 *kvo = kv_out ? kv_out + (size_t)b * N : nullptr;
  if (tile == 0) {
    // ids outside [0, K) are counted nowhere, so the counted points end before
    // N; the positions past them get -1 (key, value) instead of whatever an
    // earlier call left there.  Nothing to do when every id is valid.
    const int total = (int)(tb[bins - 1] + (uint32_t)counts[(size_t)b * bins + bins - 1]);
    for (int i = total + threadIdx.x; i < N; i += kSortThreads) {
      if (kvo) kvo[i] = make_int2(-1, -1);
      if (vo) vo[i] = -1;
      if (ko) ko[i] = -1;
    }
  }
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int r = 0; r < kRounds; ++r) {
    const unsigned dg = wk.dg[r], peers = wk.peers[r];
    uint32_t pos = 0;
    if (dg != kNoDigit) pos = cnt[dg] + __popc(peers & lt);
    __syncwarp();
    if (dg != kNoDigit) {
      if (lane == __ffs(peers) - 1) cnt[dg] += __popc(peers);
      const int32_t val = vals_in ? vals[r] : (int32_t)(base + r * 32 + lane);
      if (kvo) kvo[pos] = make_int2(wk.key[r], val);
      if (vo) vo[pos] = val;
      if (ko) ko[pos] = wk.key[r];
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

// offsets[b][k] = sum of counts[b][k'] over k' < k, one CTA per batch, any K.
__global__ void __launch_bounds__(1024) k_offsets(const int32_t *__restrict__ counts, int K,
                                                  int32_t *__restrict__ offsets) {
  __shared__ uint32_t wsum[32];
  const int b = blockIdx.x;
  const int32_t *cb = counts + (size_t)b * K;
  const int per = (K + (int)blockDim.x - 1) / (int)blockDim.x;
  const int lo = min(K, (int)threadIdx.x * per), hi = min(K, lo + per);
  uint32_t local = 0;
  for (int k = lo; k < hi; ++k) local += (uint32_t)cb[k];
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
  for (int k = lo; k < hi; ++k) {
    offsets[(size_t)b * K + k] = (int32_t)run;
    run += (uint32_t)cb[k];
  }
}

int bits_for(int K) {
  int n = 0;
  while (n < 31 && (1LL << n) < (long long)K) ++n;
  return n;
}

int set_attrs() {
  const int hist_max = kSortWarps * (1 << kMaxDigitBits) * 4;
  const int scat_max = (kSortWarps + 1) * (1 << kMaxDigitBits) * 4;
  FK_TRY(set_smem_limit((const void *)k_tile_hist, hist_max));
  FK_TRY(set_smem_limit((const void *)k_tile_scatter, scat_max));
  FK_TRY(set_smem_limit((const void *)k_count, 64 * 1024));
  return FK_OK;
}

// One counting-sort pass.  digit_counts (B, bins) receives the digit totals;
// offsets_out (B, bins), when not NULL, their exclusive scan.
int one_pass(Workspace *ws, const int32_t *keys_in, const int32_t *vals_in, int B, int N, int K,
             int T, PassCfg pc, int32_t *digit_counts, int32_t *offsets_out, int32_t *keys_out,
             int32_t *vals_out, int2 *kv_out, cudaStream_t s, bool have_hist = false) {
  FK_TRY(ensure(ws->table, (size_t)B * T * pc.bins * sizeof(uint32_t)));
  uint32_t *H = (uint32_t *)ws->table.p;
  const dim3 grid((unsigned)T, (unsigned)B);
  const size_t shm_h = (size_t)kSortWarps * pc.bins * sizeof(uint32_t);
  const size_t shm_s = (size_t)(kSortWarps + 1) * pc.bins * sizeof(uint32_t);
  if (!have_hist) {
    k_tile_hist<<<grid, kSortThreads, shm_h, s>>>(keys_in, N, K, T, pc, H, ws->err);
    FK_TRY(launched());
    FK_CUDA(cudaGetLastError());
  }
  FK_CUDA(launch_pdl(k_scan_tiles, dim3((unsigned)((pc.bins + 31) / 32), (unsigned)B), dim3(kSortThreads),
                    0, s, H, pc.bins, T, digit_counts, ws->maxshift));
  FK_TRY(launched());
  FK_CUDA(launch_pdl(k_tile_scatter, grid, dim3(kSortThreads), shm_s, s, keys_in, vals_in, N, K, T, pc, H,
                     (const int32_t *)digit_counts, offsets_out, keys_out, vals_out, kv_out,
                     have_hist ? 1 : 0, ws->err));
  FK_TRY(launched());
  return FK_OK;
}

}  // namespace

bool sort_single_pass(int K) { return bits_for(K) <= kMaxDigitBits; }

size_t sort_table_bytes(int B, long long N, int K) {
  return (size_t)B * ((N + kSortTile - 1) / kSortTile) * K * sizeof(uint32_t);
}

int run_sort_prehist(Workspace *ws, const int32_t *ids, int B, long long N_, int K, int32_t *counts,
                     int32_t *offsets, int32_t *perm, int2 *kv_out, cudaStream_t s) {
  if (!sort_single_pass(K)) return set_error(FK_EUNSUPPORTED, "fused histogram needs K <= 4096");
  FK_TRY(set_attrs());
  const int N = (int)N_;
  const int T = (int)((N_ + kSortTile - 1) / kSortTile);
  int32_t *cnt = counts, *off = offsets;
  if (!cnt) {
    FK_TRY(ensure(ws->counts, (size_t)B * K * sizeof(int32_t)));
    cnt = (int32_t *)ws->counts.p;
  }
  if (!off) {
    FK_TRY(ensure(ws->offsets, (size_t)B * K * sizeof(int32_t)));
    off = (int32_t *)ws->offsets.p;
  }
  PassCfg pc{0, 0xffffffffu, K, bits_for(K), true};
  return one_pass(ws, ids, nullptr, B, N, K, T, pc, cnt, off, nullptr, perm, kv_out, s, true);
}

int run_sort(Workspace *ws, const int32_t *ids, int B, long long N_, int K, int32_t *counts,
             int32_t *offsets, int32_t *perm, int2 *kv_out, cudaStream_t s) {
  FK_TRY(set_attrs());
  const int N = (int)N_;
  const int T = (int)((N_ + kSortTile - 1) / kSortTile);
  const int nbits = bits_for(K);
  int32_t *cnt = counts;
  if (!cnt) {
    FK_TRY(ensure(ws->counts, (size_t)B * K * sizeof(int32_t)));
    cnt = (int32_t *)ws->counts.p;
  }
  if (nbits <= kMaxDigitBits) {
    int32_t *off = offsets;
    if (!off) {
      FK_TRY(ensure(ws->offsets, (size_t)B * K * sizeof(int32_t)));
      off = (int32_t *)ws->offsets.p;
    }
    PassCfg pc{0, 0xffffffffu, K, nbits, true};
    return one_pass(ws, ids, nullptr, B, N, K, T, pc, cnt, off, nullptr, perm, kv_out, s);
  }
  const int lo = (nbits + 1) / 2, hi = nbits - lo;
  const size_t nb = (size_t)B * N * sizeof(int32_t);
  FK_TRY(ensure(ws->keys_b, nb));
  FK_TRY(ensure(ws->vals_b, nb));
  int32_t *kt = (int32_t *)ws->keys_b.p, *vt = (int32_t *)ws->vals_b.p;
  // digit totals of the passes live in the workspace (at most 4096 per batch)
  FK_TRY(ensure(ws->digit_off, (size_t)B * (1 << kMaxDigitBits) * sizeof(int32_t)));
  int32_t *dcnt = (int32_t *)ws->digit_off.p;
  PassCfg p1{0, (1u << lo) - 1u, 1 << lo, lo, true};
  FK_TRY(one_pass(ws, ids, nullptr, B, N, K, T, p1, dcnt, nullptr, kt, vt, nullptr, s));
  // the second pass validates its keys too, so the -1 entries that stand for
  // out-of-range ids past the first pass's counted points are dropped again
  PassCfg p2{lo, (1u << hi) - 1u, 1 << hi, hi, true};
  FK_TRY(one_pass(ws, kt, vt, B, N, K, T, p2, dcnt, nullptr, nullptr, perm, kv_out, s));
  // cluster counts and offsets (a pass's digit totals are not cluster totals)
  FK_CUDA(cudaMemsetAsync(cnt, 0, (size_t)B * K * sizeof(int32_t), s));
  const int use_smem = (size_t)K * 4 <= 64 * 1024 ? 1 : 0;
  k_count<<<dim3((unsigned)T, (unsigned)B), 256, use_smem ? K * 4 : 0, s>>>(ids, N, K, cnt, use_smem);
  FK_TRY(launched());
  FK_CUDA(cudaGetLastError());
  if (offsets) {
    k_offsets<<<B, 1024, 0, s>>>(cnt, K, offsets);
    FK_TRY(launched());
    FK_CUDA(cudaGetLastError());
  }
  return FK_OK;
}

}  // namespace fk
