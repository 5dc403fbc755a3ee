/*
 * Seeded synthetic inputs for the batched K-Means workloads.
 *
 * This module only makes inputs: Gaussian-mixture point sets stored in
 * fp32 / fp16 / bf16 and seed-chosen initial centroid index sets.  It holds
 * none of the clustering arithmetic; both the fp64 checker and the GPU path
 * consume its output.
 *
 * Random numbers come from a counter-based generator: the SplitMix64 output
 * function (Steele, Lea & Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014) applied to (key, counter).  Every element is a
 * pure function of (seed, batch, point, dimension), so the output does not
 * depend on the number of threads.
 *
 * Normals use the Box-Muller transform on two uniforms in (0,1).
 * Conversion to fp16 / bf16 is round-to-nearest-even, written here from the
 * IEEE-754 binary16 and bfloat16 bit layouts.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { SD_F32 = 0, SD_F16 = 1, SD_BF16 = 2 };

static inline uint64_t mix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ULL;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* One 64-bit draw for (key, counter). */
static inline uint64_t draw(uint64_t key, uint64_t ctr) {
  return mix64(key ^ mix64(ctr + 0x632BE59BD9B4E019ULL));
}

/* Uniform in the open interval (0, 1) with 53 random bits. */
static inline double unif(uint64_t key, uint64_t ctr) {
  return ((double)(draw(key, ctr) >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

static inline uint64_t key_of(uint64_t seed, uint64_t tag, uint64_t a) {
  return mix64(mix64(seed ^ (tag * 0xD1B54A32D192ED03ULL)) ^ (a * 0xA24BAED4963EE407ULL));
}

/* Two independent standard normals for (key, counter pair index). */
static inline void normal2(uint64_t key, uint64_t pair, double *z0, double *z1) {
  const double two_pi = 6.283185307179586476925286766559;
  double u1 = unif(key, 2 * pair), u2 = unif(key, 2 * pair + 1);
  double r = sqrt(-2.0 * log(u1));
  *z0 = r * cos(two_pi * u2);
  *z1 = r * sin(two_pi * u2);
}

/* float -> binary16, round to nearest even; overflow goes to +-inf. */
static uint16_t to_f16(float f) {
  uint32_t x;
  memcpy(&x, &f, 4);
  uint32_t sign = (x >> 16) & 0x8000u;
  uint32_t ex = (x >> 23) & 0xFFu;
  uint32_t man = x & 0x7FFFFFu;
  if (ex == 0xFF) return (uint16_t)(sign | 0x7C00u | (man ? 0x200u : 0));
  int e = (int)ex - 127 + 15;
  if (e >= 31) return (uint16_t)(sign | 0x7C00u);
  if (e <= 0) {
    if (e < -10) return (uint16_t)sign;
    man |= 0x800000u;
    int shift = 14 - e;
    uint32_t q = man >> shift;
    uint32_t rem = man & ((1u << shift) - 1);
    uint32_t half = 1u << (shift - 1);
    if (rem > half || (rem == half && (q & 1))) q++;
    return (uint16_t)(sign | q);
  }
  uint32_t q = ((uint32_t)e << 10) | (man >> 13);
  uint32_t rem = man & 0x1FFFu;
  if (rem > 0x1000u || (rem == 0x1000u && (q & 1))) q++; /* may carry into exponent: correct */
  return (uint16_t)(sign | q);
}

/* float -> bfloat16, round to nearest even. */
static uint16_t to_bf16(float f) {
  uint32_t x;
  memcpy(&x, &f, 4);
  if ((x & 0x7F800000u) == 0x7F800000u && (x & 0x7FFFFFu)) return (uint16_t)((x >> 16) | 0x40u);
  uint32_t lsb = (x >> 16) & 1u;
  x += 0x7FFFu + lsb;
  return (uint16_t)(x >> 16);
}

static inline void store(void *out, int dtype, size_t i, double v) {
  float f = (float)v;
  if (dtype == SD_F32) ((float *)out)[i] = f;
  else if (dtype == SD_F16) ((uint16_t *)out)[i] = to_f16(f);
  else ((uint16_t *)out)[i] = to_bf16(f);
}

/*
 * Gaussian mixture.  n_comp components with means ~ N(0, mean_std^2 I) drawn
 * once per batch, unit variance around each mean.  Component weights are equal
 * when zipf_s <= 0, else proportional to (c+1)^(-zipf_s).  n_comp == 1 with
 * mean_std == 0 gives i.i.d. N(0,1).  out is (B, N, d) row-major.
 * comp_out (nullable) receives each point's component, (B, N) int32.
 */
int synth_mixture(void *out, int dtype, int B, long long N, int d, int n_comp,
                  double mean_std, double zipf_s, uint64_t seed, int nthreads,
                  int32_t *comp_out) {
  if (!out || B <= 0 || N <= 0 || d <= 0 || n_comp <= 0) return 1;
  if (dtype < 0 || dtype > 2) return 1;
  double *means = (double *)malloc(sizeof(double) * (size_t)n_comp * (size_t)d);
  double *cdf = (double *)malloc(sizeof(double) * (size_t)n_comp);
  if (!means || !cdf) { free(means); free(cdf); return 2; }
  double tot = 0.0;
  for (int c = 0; c < n_comp; ++c) {
    double w = zipf_s > 0.0 ? pow((double)(c + 1), -zipf_s) : 1.0;
    tot += w;
    cdf[c] = tot;
  }
  for (int c = 0; c < n_comp; ++c) cdf[c] /= tot;
  cdf[n_comp - 1] = 1.0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
  for (int b = 0; b < B; ++b) {
    uint64_t kmean = key_of(seed, 1, (uint64_t)b);
    uint64_t kcomp = key_of(seed, 2, (uint64_t)b);
    uint64_t knoise = key_of(seed, 3, (uint64_t)b);
    for (int c = 0; c < n_comp; ++c) {
      for (int j = 0; j < d; j += 2) {
        double z0, z1;
        normal2(kmean, ((uint64_t)c * (uint64_t)d + (uint64_t)j) / 2, &z0, &z1);
        means[(size_t)c * d + j] = mean_std * z0;
        if (j + 1 < d) means[(size_t)c * d + j + 1] = mean_std * z1;
      }
    }
    /* pair index for noise: per point, ceil(d/2) pairs */
    const uint64_t pairs = (uint64_t)(d + 1) / 2;
#pragma omp parallel for schedule(static)
    for (long long i = 0; i < N; ++i) {
      int comp = 0;
      if (n_comp > 1) {
        double u = unif(kcomp, (uint64_t)i);
        int lo = 0, hi = n_comp - 1;
        while (lo < hi) {
          int mid = (lo + hi) / 2;
          if (u <= cdf[mid]) hi = mid; else lo = mid + 1;
        }
        comp = lo;
      }
      if (comp_out) comp_out[(size_t)b * N + i] = comp;
      const double *m = means + (size_t)comp * d;
      size_t base = ((size_t)b * (size_t)N + (size_t)i) * (size_t)d;
      for (int j = 0; j < d; j += 2) {
        double z0, z1;
        normal2(knoise, (uint64_t)i * pairs + (uint64_t)j / 2, &z0, &z1);
        store(out, dtype, base + j, m[j] + z0);
        if (j + 1 < d) store(out, dtype, base + j + 1, m[j + 1] + z1);
      }
    }
  }
  free(means);
  free(cdf);
  return 0;
}

/* Uniform integer in [0, n) from a 64-bit draw (multiply-high). */
static inline uint64_t below(uint64_t r, uint64_t n) {
  return (uint64_t)(((unsigned __int128)r * (unsigned __int128)n) >> 64);
}

/* open-addressing map int64 -> int64 for a sparse Fisher-Yates */
typedef struct { int64_t *keys; int64_t *vals; size_t cap; } i64map;

static int map_init(i64map *m, size_t want) {
  size_t cap = 16;
  while (cap < 2 * want + 16) cap <<= 1;
  m->keys = (int64_t *)malloc(cap * sizeof(int64_t));
  m->vals = (int64_t *)malloc(cap * sizeof(int64_t));
  m->cap = cap;
  if (!m->keys || !m->vals) return 1;
  for (size_t i = 0; i < cap; ++i) m->keys[i] = -1;
  return 0;
}
static size_t map_slot(const i64map *m, int64_t k) {
  size_t h = (size_t)mix64((uint64_t)k) & (m->cap - 1);
  while (m->keys[h] != -1 && m->keys[h] != k) h = (h + 1) & (m->cap - 1);
  return h;
}
static int64_t map_get(const i64map *m, int64_t k) {
  size_t h = map_slot(m, k);
  return m->keys[h] == k ? m->vals[h] : k;
}
static void map_put(i64map *m, int64_t k, int64_t v) {
  size_t h = map_slot(m, k);
  m->keys[h] = k;
  m->vals[h] = v;
}

/*
 * K distinct point indices per batch, in [0, N): the first K draws of a
 * Fisher-Yates shuffle of 0..N-1 (kept sparse, so memory is O(K)).  The batch b
 * uses seed (seed_base + b).  idx is (B, K) int64.
 */
int synth_init_indices(int64_t *idx, int B, long long N, int K, uint64_t seed_base) {
  if (!idx || B <= 0 || N <= 0 || K <= 0 || (long long)K > N) return 1;
  for (int b = 0; b < B; ++b) {
    i64map m;
    if (map_init(&m, (size_t)K * 2)) { free(m.keys); free(m.vals); return 2; }
    uint64_t key = key_of(seed_base + (uint64_t)b, 4, 0);
    for (int k = 0; k < K; ++k) {
      int64_t r = (int64_t)k + (int64_t)below(draw(key, (uint64_t)k), (uint64_t)(N - k));
      int64_t vr = map_get(&m, r), vk = map_get(&m, k);
      map_put(&m, r, vk);
      map_put(&m, k, vr);
      idx[(size_t)b * K + k] = vr;
    }
    free(m.keys);
    free(m.vals);
  }
  return 0;
}

/* Rows x[b, idx[b,k], :] -> out[b, k, :]; element size esz bytes. */
int synth_gather_rows(const void *x, int esz, int B, long long N, int d, const int64_t *idx,
                      int K, void *out) {
  if (!x || !idx || !out || esz <= 0) return 1;
  size_t row = (size_t)d * (size_t)esz;
  for (int b = 0; b < B; ++b)
    for (int k = 0; k < K; ++k) {
      int64_t i = idx[(size_t)b * K + k];
      if (i < 0 || i >= N) return 1;
      memcpy((char *)out + ((size_t)b * K + k) * row,
             (const char *)x + ((size_t)b * (size_t)N + (size_t)i) * row, row);
    }
  return 0;
}
