/*
 * fp64 reference for batched Lloyd's K-Means.  TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg load
 * this library.  The CUDA library never calls it and shares no code with it.
 *
 * What it computes is the plain definition of one Lloyd iteration, written out
 * step by step in double precision:
 *
 *   assign  id[b,i] = argmin_k  sum_j (x[b,i,j] - c^[b,k,j])^2
 *           (ties -> lowest k), where c^ is the centroid rounded to the
 *           input dtype when a dtype is given.  Squared Euclidean distance is
 *           the reading of "distance computation" in "Flash-KMeans: Fast and
 *           Memory-Efficient Exact K-Means" (Abstract) and in the paper
 *           summary "Flash-KMeans: IO感知的精确K-Means" (section
 *           "什么是 Flash-KMeans": assignment computes each point's distance
 *           to every centroid and picks the nearest one).  The method's
 *           ||c||^2 - 2 x.c form has the same argmin; the direct form is kept
 *           here so exact ties are exact.
 *   update  counts[b,k] = #{i : id = k};  new[b,k] = mean of its points, and
 *           an empty cluster keeps its previous centroid (the pages are
 *           silent; this reading is fixed for the build).  Same section: the
 *           update averages the points of each cluster into its new centroid.
 *   sort    perm[b,:] = point indices ordered by (id, i) -- the inverse
 *           mapping that the sort-inverse update builds by sorting the
 *           assignment vector ("Flash-KMeans: IO感知的精确K-Means", section
 *           "它攻克的兩大瓶頸", the paragraph on Sort-Inverse Update).  The
 *           pair key is unique, so the order is fully defined.
 *   shift   max over b,k of ||new - old||_2; the Lloyd loop stops once it is
 *           below tol (strict), or after max_iter iterations.  The tol
 *           argument appears in the functional API example of "flash-kmeans
 *           and the return of exact K-Means on the GPU" (section "Exact
 *           K-Means, with the assignment step written in Triton").
 *
 * Inputs x arrive in their storage dtype (fp32 / fp16 / bf16) and are widened
 * exactly to double.  Rounding of centroids to fp16 / bf16 is round to nearest
 * even, written from the binary16 / bfloat16 definitions with rint().
 *
 * A mutation switch plants known mistakes; the pin tests use it to show that
 * each planted mistake is caught.  It is off (0) unless a test sets it.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_F16 = 1, OR_BF16 = 2, OR_NOROUND = -1 };

static int g_mutation = 0;
void or_set_mutation(int m) { g_mutation = m; }
int or_get_mutation(void) { return g_mutation; }

static void set_threads(int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
}

int or_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ---------------------------------------------------------------- widening */

static double half_to_double(uint16_t h) {
  int sign = (h >> 15) & 1, ex = (h >> 10) & 31, man = h & 1023;
  double v;
  if (ex == 0) v = ldexp((double)man, -24);               /* subnormal / zero */
  else if (ex == 31) v = man ? NAN : INFINITY;
  else v = ldexp((double)(1024 + man), ex - 25);            /* (1.man) * 2^(ex-15) */
  return sign ? -v : v;
}

/* All 65536 binary16 values, widened once by half_to_double at load time. */
static double g_half_table[65536];

__attribute__((constructor)) static void build_half_table(void) {
  for (uint32_t h = 0; h < 65536u; ++h) g_half_table[h] = half_to_double((uint16_t)h);
}

static double bf16_to_double(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

static inline double load_x(const void *x, int dtype, size_t i) {
  if (dtype == OR_F32) return (double)((const float *)x)[i];
  if (dtype == OR_F16) return g_half_table[((const uint16_t *)x)[i]];
  return bf16_to_double(((const uint16_t *)x)[i]);
}

/* Widen n stored values to double (exact). */
int or_widen(const void *x, int dtype, long long n, double *out) {
  if (!x || !out || n < 0) return 1;
  for (long long i = 0; i < n; ++i) out[i] = load_x(x, dtype, (size_t)i);
  return 0;
}

/* -------------------------------------------------------------- rounding */

/* Round v to a binary floating format with p significand bits, minimum normal
 * exponent emin and largest finite value maxf; round half to even. */
static double round_format(double v, int p, int emin, double maxf) {
  if (v == 0.0 || !isfinite(v)) return v;
  double a = fabs(v);
  int e;
  frexp(a, &e);             /* a = m * 2^e, m in [0.5, 1) -> a in [2^(e-1), 2^e) */
  int ex = e - 1;           /* a in [2^ex, 2^(ex+1)) */
  if (ex < emin) ex = emin; /* subnormal range has the quantum of the smallest normal binade */
  double q = ldexp(1.0, ex - (p - 1));
  double r = rint(a / q) * q; /* a/q is exact; rint rounds half to even */
  if (r > maxf) r = INFINITY;
  return v < 0 ? -r : r;
}

double or_round_value(double v, int dtype) {
  if (dtype == OR_F32) return (double)(float)v;
  if (dtype == OR_F16) return round_format(v, 11, -14, 65504.0);
  if (dtype == OR_BF16) return round_format(v, 8, -126, ldexp(255.0, 120)); /* (2-2^-7)*2^127 */
  return v;
}

int or_round(const double *c, long long n, int dtype, double *out) {
  if (!c || !out) return 1;
  for (long long i = 0; i < n; ++i) out[i] = or_round_value(c[i], dtype);
  return 0;
}

/* ---------------------------------------------------------------- assign */

static double sqdist(const void *x, int dtype, size_t xrow, const double *c, int d) {
  double s = 0.0;
  int dd = (g_mutation == 4) ? d - 1 : d; /* planted: drops the last dimension */
  for (int j = 0; j < dd; ++j) {
    double xj = load_x(x, dtype, xrow + (size_t)j);
    double t = (g_mutation == 7) ? xj + c[j] : xj - c[j]; /* planted: wrong sign */
    s += t * t;
  }
  return s;
}

/*
 * ids[b,i] = argmin_k ||x[b,i] - chat[b,k]||^2, lowest k on ties.
 * gap[b,i] (nullable) = second-smallest minus smallest squared distance
 * (+inf when K == 1).  dmin (nullable) = the smallest squared distance.
 * chat is used as given (callers round it first when they mirror a dtype).
 */
int or_assign(const void *x, int dtype, const double *chat, int B, long long N, int K, int d,
              int32_t *ids, double *gap, double *dmin, int nthreads) {
  if (!x || !chat || !ids || B <= 0 || N <= 0 || K <= 0 || d <= 0) return 1;
  set_threads(nthreads);
  for (int b = 0; b < B; ++b) {
    const double *cb = chat + (size_t)b * K * d;
#pragma omp parallel for schedule(dynamic, 64)
    for (long long i = 0; i < N; ++i) {
      size_t xrow = ((size_t)b * (size_t)N + (size_t)i) * (size_t)d;
      double best = INFINITY, second = INFINITY;
      int arg = 0;
      for (int k = 0; k < K; ++k) {
        const double *ck = (g_mutation == 8) ? cb + (size_t)k : cb + (size_t)k * d;
        double dist;
        if (g_mutation == 8) { /* planted: transposed centroid operand (stride K) */
          dist = 0.0;
          for (int j = 0; j < d; ++j) {
            size_t off = (size_t)j * K;
            double cj = (off < (size_t)K * d) ? ck[off] : 0.0;
            double t = load_x(x, dtype, xrow + (size_t)j) - cj;
            dist += t * t;
          }
        } else {
          dist = sqdist(x, dtype, xrow, ck, d);
        }
        int better = (g_mutation == 1) ? (dist <= best) : (dist < best); /* planted: ties -> highest k */
        if (better) {
          second = best;
          best = dist;
          arg = k;
        } else if (dist < second) {
          second = dist;
        }
      }
      ids[(size_t)b * N + i] = arg;
      if (gap) gap[(size_t)b * N + i] = second - best;
      if (dmin) dmin[(size_t)b * N + i] = best;
    }
  }
  return 0;
}

/* ------------------------------------------------------------------ sort */

typedef struct { int32_t id; int64_t i; } key_t_;

static int cmp_key(const void *a, const void *b) {
  const key_t_ *p = (const key_t_ *)a, *q = (const key_t_ *)b;
  if (p->id != q->id) return p->id < q->id ? -1 : 1;
  if (p->i != q->i) {
    int asc = p->i < q->i ? -1 : 1;
    return g_mutation == 5 ? -asc : asc; /* planted: descending index inside a cluster */
  }
  return 0;
}

/* counts[b,k] and perm[b,:] (indices ordered by (id, i)).  Either output may be null. */
int or_sort(const int32_t *ids, int B, long long N, int K, int64_t *counts, int64_t *perm) {
  if (!ids || B <= 0 || N <= 0 || K <= 0) return 1;
  for (int b = 0; b < B; ++b) {
    const int32_t *ib = ids + (size_t)b * N;
    for (long long i = 0; i < N; ++i)
      if (ib[i] < 0 || ib[i] >= K) return 2;
    if (counts) {
      int64_t *cb = counts + (size_t)b * K;
      for (int k = 0; k < K; ++k) cb[k] = 0;
      for (long long i = 0; i < N; ++i) cb[ib[i]]++;
      if (g_mutation == 9) cb[0] += 1; /* planted: miscounted cluster 0 */
    }
    if (perm) {
      key_t_ *keys = (key_t_ *)malloc(sizeof(key_t_) * (size_t)N);
      if (!keys) return 3;
      for (long long i = 0; i < N; ++i) { keys[i].id = ib[i]; keys[i].i = i; }
      qsort(keys, (size_t)N, sizeof(key_t_), cmp_key);
      for (long long j = 0; j < N; ++j) perm[(size_t)b * N + j] = keys[j].i;
      free(keys);
    }
  }
  return 0;
}

/* ---------------------------------------------------------------- update */

/*
 * new_c[b,k] = mean of the points with id k (summed in increasing i), or
 * old_c[b,k] when the cluster is empty.  counts (nullable) gets the sizes.
 * shift (nullable, B*K) gets ||new - old||_2; maxshift (nullable) the max.
 */
int or_update(const void *x, int dtype, const int32_t *ids, int B, long long N, int K, int d,
              const double *old_c, double *new_c, int64_t *counts, double *shift,
              double *maxshift) {
  if (!x || !ids || !old_c || !new_c || B <= 0 || N <= 0 || K <= 0 || d <= 0) return 1;
  for (size_t i = 0; i < (size_t)B * (size_t)N; ++i)
    if (ids[i] < 0 || ids[i] >= K) return 2;
  double mx = 0.0;
  int rc = 0;
  /* batches are independent problems; each thread owns whole batches */
#pragma omp parallel for schedule(dynamic, 1) reduction(max : mx)
  for (int b = 0; b < B; ++b) {
    double *sum = (double *)calloc((size_t)K * d, sizeof(double));
    int64_t *cnt = (int64_t *)calloc((size_t)K, sizeof(int64_t));
    if (!sum || !cnt) {
      free(sum);
      free(cnt);
#pragma omp atomic write
      rc = 3;
      continue;
    }
    for (long long i = 0; i < N; ++i) {
      int32_t k = ids[(size_t)b * N + i];
      cnt[k]++;
      size_t xrow = ((size_t)b * (size_t)N + (size_t)i) * (size_t)d;
      double *s = sum + (size_t)k * d;
      for (int j = 0; j < d; ++j) s[j] += load_x(x, dtype, xrow + (size_t)j);
    }
    for (int k = 0; k < K; ++k) {
      const double *o = old_c + ((size_t)b * K + k) * d;
      double *n = new_c + ((size_t)b * K + k) * d;
      double s2 = 0.0;
      for (int j = 0; j < d; ++j) {
        double v;
        if (cnt[k] > 0) {
          double den = (double)cnt[k] + (g_mutation == 3 ? 1.0 : 0.0); /* planted: count + 1 */
          v = sum[(size_t)k * d + j] / den;
        } else {
          v = (g_mutation == 2) ? 0.0 : o[j]; /* planted: empty cluster zeroed */
        }
        double t = v - o[j];
        s2 += (g_mutation == 6) ? fabs(t) : t * t; /* planted: L1-style shift */
        n[j] = v;
      }
      double sh = (g_mutation == 6) ? s2 : sqrt(s2);
      if (shift) shift[(size_t)b * K + k] = sh;
      if (sh > mx) mx = sh;
      if (counts) counts[(size_t)b * K + k] = cnt[k] + ((g_mutation == 9 && k == 0) ? 1 : 0);
    }
    free(sum);
    free(cnt);
  }
  if (maxshift) *maxshift = mx;
  return rc;
}

/* sum over b,i of ||x[b,i] - c[b,id]||^2 (squared error objective). */
double or_objective(const void *x, int dtype, const double *c, const int32_t *ids, int B,
                    long long N, int K, int d) {
  double tot = 0.0;
  for (int b = 0; b < B; ++b)
    for (long long i = 0; i < N; ++i) {
      int32_t k = ids[(size_t)b * N + i];
      size_t xrow = ((size_t)b * (size_t)N + (size_t)i) * (size_t)d;
      const double *ck = c + ((size_t)b * K + k) * d;
      double s = 0.0;
      for (int j = 0; j < d; ++j) {
        double t = load_x(x, dtype, xrow + (size_t)j) - ck[j];
        s += t * t;
      }
      tot += s;
    }
  return tot;
}

/*
 * The Lloyd loop.  centers holds the initial centroids on entry (double) and
 * the centroids of the last update on exit; ids holds the last assignment.
 * round_dtype: centroids are rounded to this dtype before each assign
 * (OR_NOROUND = -1 keeps them exact).  obj_trace (nullable, max_iter) gets
 * the objective of each assignment against the centroids it used.
 */
int or_lloyd(const void *x, int dtype, int B, long long N, int K, int d, int round_dtype,
             int max_iter, double tol, int32_t *ids, double *centers, int64_t *counts,
             int *iters_run, double *last_maxshift, double *obj_trace, int nthreads) {
  if (!x || !centers || !ids || max_iter < 0) return 1;
  size_t nc = (size_t)B * K * d;
  double *chat = (double *)malloc(nc * sizeof(double));
  double *next = (double *)malloc(nc * sizeof(double));
  if (!chat || !next) { free(chat); free(next); return 3; }
  int it = 0;
  double ms = 0.0;
  int rc = 0;
  for (it = 0; it < max_iter; ++it) {
    if (round_dtype == OR_NOROUND) memcpy(chat, centers, nc * sizeof(double));
    else or_round(centers, (long long)nc, round_dtype, chat);
    rc = or_assign(x, dtype, chat, B, N, K, d, ids, NULL, NULL, nthreads);
    if (rc) break;
    if (obj_trace) obj_trace[it] = or_objective(x, dtype, chat, ids, B, N, K, d);
    rc = or_update(x, dtype, ids, B, N, K, d, centers, next, counts, NULL, &ms);
    if (rc) break;
    memcpy(centers, next, nc * sizeof(double));
    if (ms < tol) { ++it; break; }
  }
  free(chat);
  free(next);
  if (iters_run) *iters_run = it;
  if (last_maxshift) *last_maxshift = ms;
  return rc;
}
