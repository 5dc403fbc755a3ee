/*
 * fk.h -- C ABI of libfk.so: exact batched Lloyd's K-Means on one NVIDIA
 * B200 (sm_100a).
 *
 * The library implements the two kernel-level ideas of flash-kmeans:
 *   - FlashAssign: the point-to-centroid distance is fused with a running
 *     argmin, so the (B, N, K) distance matrix never exists
 *     ("Flash-KMeans: Fast and Memory-Efficient Exact K-Means", Abstract;
 *     "flash-kmeans and the return of exact K-Means on the GPU", section
 *     "The point of the kernel is that the distance matrix never exists").
 *   - Sort-inverse update: the assignment vector is sorted by cluster id
 *     (a stable counting sort here), each contiguous segment is reduced on
 *     chip and flushed with one atomic add per segment piece
 *     ("Flash-KMeans: IO感知的精确K-Means", section "它攻克的兩大瓶頸").
 * plus the chunked host-to-device stream overlap for point sets held in
 * pinned host memory (same Abstract; "flash-kmeans and the return of exact
 * K-Means on the GPU", section "Multi-GPU scaling without a NCCL
 * dependency", the double-buffered host-to-device pipeline).
 *
 * Conventions shared by every entry point
 *   - Layouts are dense row-major: points x (B, N, d), centroids (B, K, d),
 *     ids (B, N), counts / offsets (B, K), perm (B, N).  d is contiguous.
 *   - dtype is one of FK_F32, FK_F16, FK_BF16 and describes x and any
 *     centroid tensor passed "in x's dtype".  Accumulation is fp32.
 *   - Pointers are device pointers unless stated otherwise.  The caller owns
 *     every buffer it passes.  The library keeps its own scratch (workspace)
 *     per (device, stream), allocated on first use and grown as needed;
 *     fk_release() frees it.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; 0 = legacy default
 *     stream) unless stated otherwise.
 *   - Every call returns an fk_status.  Nothing throws across the ABI.
 *     FK_EINVAL: a size <= 0, K > N, N or K beyond 2^31-1, a null pointer,
 *     an unknown dtype, or (fp16 / bf16) d*2 not a multiple of 16 bytes or a
 *     pointer not 16-byte aligned; also a pointer documented as device memory
 *     that is host memory or memory of another device than the current one
 *     (device memory passed where host memory is allowed must be the current
 *     device's too; managed memory is accepted).  FK_EUNSUPPORTED: a shape beyond the
 *     limits stated per call.  FK_ECUDA: a CUDA runtime error (see
 *     fk_last_error()).  FK_ETIMEOUT: a kernel's bounded wait expired (the
 *     kernel recorded it in the device error word and returned; see
 *     fk_device_error()).
 *   - Ties in the argmin go to the lowest centroid index.  An empty cluster
 *     keeps its previous centroid.
 */
#ifndef FK_H
#define FK_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *fk_stream_t; /* identical to cudaStream_t */

typedef enum { FK_F32 = 0, FK_F16 = 1, FK_BF16 = 2 } fk_dtype;

typedef enum {
  FK_OK = 0,
  FK_EINVAL = 1,
  FK_ENOMEM = 2,
  FK_ECUDA = 3,
  FK_ETIMEOUT = 4,
  FK_EUNSUPPORTED = 5
} fk_status;

/* Problem shape for fk_lloyd. */
typedef struct {
  int B;       /* independent problems (batches) */
  long long N; /* points per batch, 1 <= N <= 2^31-1 */
  int K;       /* centroids per batch, 1 <= K <= min(N, 2^24) */
  int d;       /* dimensions */
  int dtype;   /* fk_dtype of x and init_centers */
} fk_shape;

/* Where fk_lloyd keeps points that arrive in host memory. */
typedef enum {
  FK_HOST_AUTO = 0,     /* resident copy when it fits in free device memory, else streamed */
  FK_HOST_RESIDENT = 1, /* copy x to the device once, iterate there */
  FK_HOST_STREAM = 2    /* re-stream x in chunks every iteration (out-of-core path) */
} fk_host_mode;

typedef struct {
  int host_mode;          /* fk_host_mode; used only when x is host memory */
  long long chunk_points; /* streamed path: points per chunk; 0 = FK_CHUNK_POINTS
                             from the environment, else 2^24 */
  int verbose;            /* 1: one line per iteration on stderr (also with
                             FK_VERBOSE=1 in the environment) */
} fk_options;

/*
 * fk_assign -- FlashAssign (step a1).
 * ids[b,i] = argmin_k ( ||c[b,k]||^2 - 2 x[b,i].c[b,k] ), fp32 accumulation,
 * lowest k on ties; the (B, N, K) distance matrix is never written.
 * Passage: "Flash-KMeans: Fast and Memory-Efficient Exact K-Means", Abstract
 * (FlashAssign fuses distance computation with an online argmin);
 * "flash-kmeans and the return of exact K-Means on the GPU", section "The
 * point of the kernel is that the distance matrix never exists" (point tiles
 * and centroid chunks streamed on chip).
 *   x    (B, N, d) in dtype, device.  c (B, K, d) in dtype, device.
 *   ids  (B, N) int32 out, device.
 * fp16 / bf16 run on tcgen05 tensor cores (TMA-fed tiles, TMEM accumulators);
 * the squared norms enter the accumulator through one extra K = 16 MMA step,
 * so the ranking value is ||x - c||^2 (+ a per-point constant) in fp32.  For
 * d <= 128 the argmin keeps the column in the low byte of that fp32 value:
 * values within 2^-15 of each other (relative) count as tied and the lowest
 * k wins.  fp16 inputs need ||c||^2 and ||x||^2 below 2^32; beyond that the
 * device error word records FK_EUNSUPPORTED (fk_device_error()).
 * fp32 runs on CUDA cores and evaluates sum_j (x_j - c_j)^2 directly (same
 * argmin, no cancellation).
 */
int fk_assign(const void *x, const void *c, int B, long long N, int K, int d, int dtype,
              int32_t *ids, fk_stream_t stream);

/*
 * fk_update -- sort-inverse centroid update (steps a2-a5).
 * counts[b,k] = #{i : ids[b,i] = k};  centers[b,k] = mean of its points in
 * fp32, or unchanged when counts[b,k] = 0.  The points are gathered in
 * sorted order without being permuted; each segment piece is reduced on chip
 * and stored once (no atomics: a segment spread over several pieces is summed
 * in piece order by the finalize), so the result is bit-reproducible.
 * Passage: "Flash-KMeans: IO感知的精确K-Means", section "它攻克的兩大瓶頸"
 * (argsort of the assignment vector, contiguous segments, one atomic add per
 * segment); "Flash-KMeans: Fast and Memory-Efficient Exact K-Means",
 * Abstract (explicit inverse mapping).
 *   x        (B, N, d) in dtype, device.  ids (B, N) int32 in [0, K), device.
 *   centers  (B, K, d) fp32, device, in: previous centroids, out: new ones.
 *   counts   (B, K) int32 out, device; may be NULL.
 *   max_shift  nullable device float: max over b,k of ||new - old||_2.
 * ids outside [0, K) are a caller error: they are counted nowhere and the
 * device error word records FK_EINVAL (read it with fk_device_error()).
 */
int fk_update(const void *x, const int32_t *ids, int B, long long N, int K, int d,
              float *centers, int32_t *counts, fk_stream_t stream, int dtype, float *max_shift);

/*
 * fk_sort -- the stable counting sort inside fk_update (steps a2-a4),
 * exposed on its own.
 * counts[b,k] = #{i : ids[b,i] = k};  offsets[b,k] = sum_{k'<k} counts[b,k'];
 * perm[b, offsets[b,id] + r] = i where r counts the earlier points of the
 * same batch with the same id (so perm lists point indices ordered by
 * (id, index)).
 * Passage: "Flash-KMeans: IO感知的精确K-Means", section "它攻克的兩大瓶頸"
 * (sort the assignment vector by cluster id into contiguous segments).
 *   ids (B, N) int32 in [0, K), device.  counts, offsets (B, K) int32 out,
 *   device, each may be NULL.  perm (B, N) int32 out, device.
 * ids outside [0, K) are a caller error: they are counted nowhere, the
 * entries of perm past a batch's counted points are -1, and the device error
 * word records FK_EINVAL.
 */
int fk_sort(const int32_t *ids, int B, long long N, int K, int32_t *counts, int32_t *offsets,
            int32_t *perm, fk_stream_t stream);

/*
 * fk_lloyd -- the Lloyd loop (steps a1-a7).
 * Initial centroids are init_centers (the caller picks them, e.g. a seeded
 * index set of points).  Each iteration assigns every point, then updates
 * the centroids; after iteration t the loop stops when the max centroid
 * shift is below tol (strict: tol <= 0 always runs max_iter iterations).
 * On return ids holds the last assignment and centers the centroids of the
 * last update.  The fp32 centroids are rounded to dtype (nearest even)
 * before each assign.
 * Passage: "flash-kmeans and the return of exact K-Means on the GPU",
 * section "Exact K-Means, with the assignment step written in Triton"
 * (batch_kmeans_Euclid(x, n_clusters, tol, verbose) returning ids and
 * centers); "Flash-KMeans: IO感知的精确K-Means", section "什么是 Flash-KMeans"
 * (one Lloyd iteration = assign + update, exact).
 *   x             (B, N, d) in dtype: device memory, or host memory
 *                 (pinned for overlap); see fk_options.host_mode.
 *   init_centers  (B, K, d) in dtype, device or host.
 *   ids           (B, N) int32 out, device or host.
 *   centers       (B, K, d) fp32 out, device or host.
 *   iters_run     nullable host int: iterations executed.
 *   opts          nullable: defaults {FK_HOST_AUTO, 2^24, 0}.
 * fk_lloyd synchronizes `stream` before returning and reports any device
 * error word.  Streamed mode keeps two chunk buffers on the device and
 * overlaps the copy of the next chunk with the compute of this one.
 */
int fk_lloyd(const fk_shape *shape, const void *x, const void *init_centers, int max_iter,
             float tol, int32_t *ids, float *centers, fk_stream_t stream, int *iters_run,
             const fk_options *opts);

/*
 * Data-parallel Lloyd over point blocks (one block of points per rank).
 * The pages' large-N path splits the N points of a batch into contiguous
 * blocks, one per GPU; every GPU runs its own assign and partial update,
 * the partial centroid sums and counts are summed across the GPUs, and every
 * GPU then divides ("flash-kmeans and the return of exact K-Means on the
 * GPU", section "Multi-GPU scaling without a NCCL dependency": contiguous
 * block partitions, per-GPU double-buffered pipelines, reduction of the
 * partial sums and counts).  These four calls are the per-rank pieces; the
 * exchange between them (an all-reduce of `sums` and `counts`) belongs to
 * the caller's communication layer.  One iteration on every rank:
 *     fk_lloyd_step_partial(block, centers_dt) -> ids, sums, counts
 *     sum sums and counts over the ranks
 *     fk_update_finalize(sums, counts) -> centers, centers_dt, max_shift
 * With identical totals every rank computes identical centroids.
 */

/*
 * fk_point_norms -- xn[b,i] = ||x[b,i]||^2 in fp32 (fp16 / bf16 points):
 * the point-side term the tensor-core assign ranks with.  The points of a
 * Lloyd run do not change, so a caller computes them once and passes them
 * to every fk_lloyd_step_partial on the same points.
 *   x (B, N, d) in dtype, device.  xn (B, N) fp32 out, device.
 *   fp32 points: FK_EUNSUPPORTED (that assign does not use them).
 */
int fk_point_norms(const void *x, int B, long long N, int d, int dtype, float *xn,
                   fk_stream_t stream);

/*
 * fk_init_centers -- centers[b,k,:] = init[b,k,:] widened to fp32 (exact):
 * the fp32 master copy the first fk_update_finalize starts from.
 *   init (B, K, d) in dtype, device.  centers (B, K, d) fp32 out, device.
 */
int fk_init_centers(const void *init, int B, int K, int d, int dtype, float *centers,
                    fk_stream_t stream);

/*
 * fk_lloyd_step_partial -- the local half of one data-parallel Lloyd
 * iteration on this rank's block of points: ids = FlashAssign(x, centers_dt)
 * (step a1, as fk_assign), then the sort-inverse reduction of the block
 * without the division (steps a2-a5): sums[b,k,:] = sum of the block's points
 * with id k (fp32), counts[b,k] = their number; an empty cluster gets zeros.
 *   shape       the block: N = this rank's points per batch.  N may be
 *               below K (clusters without points in the block get zeros)
 *               or 0 (an empty block: zero sums and counts; x, xn and ids
 *               are not read and may be NULL).
 *   x           (B, N, d) in dtype: device memory, or pinned host memory
 *               (then streamed in chunks of opts->chunk_points, double-
 *               buffered, as fk_lloyd's streamed mode).
 *   xn          nullable (B, N) fp32, device: fk_point_norms of x (used for
 *               device-resident fp16 / bf16 points: with d <= 128 the assign
 *               ranks with them, with d > 128 its far-point check reads them
 *               instead of re-reading rows; else ignored).
 *   centers_dt  (B, K, d) in dtype, device: the centroids to assign against
 *               (for fp32 the fp32 centroids themselves).
 *   ids         (B, N) int32 out, device.
 *   sums        (B, K, d) fp32 out, device.  counts (B, K) int32 out, device.
 *   opts        nullable; only chunk_points is read.
 * Pageable host x returns FK_EINVAL.  The call is asynchronous.
 */
int fk_lloyd_step_partial(const fk_shape *shape, const void *x, const float *xn,
                          const void *centers_dt, int32_t *ids, float *sums, int32_t *counts,
                          fk_stream_t stream, const fk_options *opts);

/*
 * fk_update_finalize -- the division of the update from summed partials:
 * centers[b,k] = sums[b,k] / counts[b,k] where counts[b,k] > 0, else
 * unchanged; centers_dt receives the centroids rounded to dtype (nearest
 * even) for the next assign; max_shift = max over b,k of ||new - old||_2.
 *   sums (B, K, d) fp32, counts (B, K) int32, device (totals over the ranks).
 *   centers     (B, K, d) fp32, device, in: previous centroids, out: new.
 *   centers_dt  (B, K, d) in dtype, device, out (ignored, may be NULL, for fp32).
 *   max_shift   nullable device float.
 */
int fk_update_finalize(const float *sums, const int32_t *counts, int B, int K, int d, int dtype,
                       float *centers, void *centers_dt, float *max_shift, fk_stream_t stream);

/*
 * fk_assign_noalloc -- fk_assign for callers that cannot allocate device
 * memory (no counterpart in the paper; it is an interface addition).
 * Same arguments, layouts and shape rules as fk_assign.  fp16 / bf16 run the
 * same kernel as fk_assign and return the same ids.  fp32 always runs the
 * CUDA-core kernel here (sum_j (x_j - c_j)^2 directly), while fk_assign moves
 * fp32 problems with d % 4 == 0 and K * d >= 16384 to the 3xTF32 tensor-core
 * path, whose scratch (a widened copy of the points) this call cannot hold;
 * on those shapes the two calls may pick different ids for points whose two
 * nearest centroids lie within 1e-3 ||x||^2 of each other (a near tie), and
 * this call is much slower.  Callers that run under an
 * allocator owning all device memory, or in loops where allocation (and the
 * synchronization a cudaFree can bring) is not allowed, cannot let fk_assign
 * grow its workspace; this call allocates nothing.  Its scratch (the
 * centroid norm rows, 32 bytes per centroid, and the kernel error word) is
 * one static device array of 4 MiB + 256 bytes that every GPU loading the
 * library holds until the process exits.
 *   Limit: B * Kpad <= 131072 for fp16 / bf16, Kpad = K rounded up to a
 *   multiple of 256; larger shapes return FK_EUNSUPPORTED.  fp32 needs no
 *   scratch and has no such limit.
 *   Unlike the other calls, this one does not check that x, c and ids are
 *   memory of the current device (it makes no runtime query that a stream
 *   capture might refuse): the caller guarantees it.
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   before any stream capture.
 *   All calls on a device share the array: calls that overlap on the GPU
 *   (e.g. on two streams) race and may return wrong ids.  The error word is
 *   cleared at the start of each call.  What the kernels record there (a
 *   bounded-wait timeout, or an fp16 squared norm of 2^32 or more: a
 *   centroid or point with ||v|| >= 65536, where the ids are unreliable) is
 *   not reported by this call, which does not synchronize, nor by
 *   fk_device_error(): read it with fk_noalloc_device_error().  Callers
 *   whose fp16 data may reach that range can also use bf16 (whose norm
 *   digits have the fp32 range).
 */
int fk_assign_noalloc(const void *x, const void *c, int B, long long N, int K, int d, int dtype,
                      int32_t *ids, fk_stream_t stream);

/*
 * fk_noalloc_device_error -- the error word of fk_assign_noalloc's static
 * scratch on the current device (an interface addition, like that call).
 * Synchronizes `stream`, reads the word and clears it with blocking copies;
 * allocates nothing.  It reports what the fk_assign_noalloc calls since the
 * last clear recorded (each call also clears the word when it starts), so
 * call it after the call whose result matters, with no other such call in
 * flight on the device.  Returns FK_OK, FK_ETIMEOUT (a bounded wait in a
 * kernel gave up) or FK_EUNSUPPORTED (an fp16 squared norm of 2^32 or
 * more: that call's ids are unreliable).
 */
int fk_noalloc_device_error(fk_stream_t stream);

/* Static text for a status code. */
const char *fk_status_string(int status);

/* Text of the last FK_ECUDA / FK_EINVAL detail recorded by this thread. */
const char *fk_last_error(void);

/*
 * Synchronizes `stream`, reads and clears the device error word of its
 * workspace.  Returns FK_OK, FK_ETIMEOUT (a bounded wait in a kernel gave
 * up), FK_EUNSUPPORTED (an fp16 squared norm of 2^32 or more reached the
 * tensor-core assign's norm digits) or FK_EINVAL (an id outside [0, K)
 * reached fk_update / fk_sort).
 */
int fk_device_error(fk_stream_t stream);

/*
 * fk_selftest_bounded_wait -- a check of the failure path, not part of the
 * method (the pages have no counterpart).  Launches one CTA that waits on an
 * mbarrier nothing ever arrives at, with the same bounded wait loop as the
 * tcgen05 kernels but a limit of limit_ns nanoseconds (0 < limit_ns <= 1e10).
 * Returns FK_ETIMEOUT (read from the device error word, which is then clear)
 * when the bounded wait works; the CUDA context stays usable.
 */
int fk_selftest_bounded_wait(long long limit_ns, fk_stream_t stream);

/*
 * fk_inject_fault -- host-side fault injection for tests of the error paths
 * (an interface addition; the pages have no counterpart).  Arms one failure
 * that fires once, at the nth occurrence of its kind, without faulting any
 * GPU:
 *   FK_FAULT_ALLOC   a workspace allocation returns FK_ENOMEM,
 *   FK_FAULT_H2D     a host-to-device copy of fk_lloyd (the resident upload,
 *                    the initial centroids, a streamed chunk) returns FK_ECUDA
 *                    before it is issued,
 *   FK_FAULT_LAUNCH  the call that launched a kernel returns FK_ECUDA right
 *                    after the launch (the kernel itself runs).
 * FK_FAULT_NONE disarms.  The environment variable FK_FAULT=alloc|h2d|launch[:n]
 * arms the same at the first check.  nth >= 1; FK_EINVAL otherwise.
 */
typedef enum { FK_FAULT_NONE = 0, FK_FAULT_ALLOC = 1, FK_FAULT_H2D = 2, FK_FAULT_LAUNCH = 3 } fk_fault;
int fk_inject_fault(int kind, long long nth);

/* Frees every workspace of the current device (no call may be in flight). */
int fk_release(void);

/* Per-phase device time, measured with CUDA events on the launching stream. */
typedef struct {
  double assign_ms;   /* FlashAssign / fp32 assign kernels */
  long long assign_launches;
  double sort_ms;     /* counting sort kernels of the update */
  double reduce_ms;   /* segment-reduce kernel */
  double finalize_ms; /* divide / shift / dtype copy kernel */
  long long update_calls;
  long long kernel_launches; /* every kernel this library launched while enabled */
  double update_ms;   /* whole update calls (sort + reduce + finalize, gaps included) */
} fk_profile;

/* Event timing: 0 off (default), 1 every phase (assign, sort, reduce,
 * finalize, whole update), 2 light (assign and whole update only: two event
 * pairs per Lloyd iteration), 3 as 2 plus a timeline of the streamed
 * pipeline's chunks (fk_profile_timeline). */
int fk_profile_enable(int on);

/*
 * fk_profile_timeline -- the chunks streamed while the level was 3, in issue
 * order: six doubles per chunk, {chunk number, device buffer (0 or 1),
 * copy begin, copy end (on the copy stream), compute begin, compute end (on
 * the compute stream: assign, sort and segment reduce of the chunk)}, times
 * in ms from the first chunk's copy begin.  Writes at most max_chunks rows to
 * out (host; NULL discards them) and their number to *rows (host, nullable),
 * synchronizes the recorded events and clears the record.  At most 65536
 * chunks are kept between two reads (later ones are not recorded); a chunk
 * whose copy began before level 3 was set is not recorded.  FK_EINVAL for
 * max_chunks < 0.  It measures the chunked host-to-device overlap
 * ("Flash-KMeans: Fast and Memory-Efficient Exact K-Means", Abstract:
 * chunked-stream overlap); an interface addition, the pages show no timeline.
 */
int fk_profile_timeline(double *out, int max_chunks, int *rows);

/* Synchronizes the recorded events, fills *out, and clears the totals if reset != 0. */
int fk_profile_read(fk_profile *out, int reset);

/* Count of kernel launches issued by this library since load. */
long long fk_launch_count(void);

/* Library version: major * 10000 + minor * 100 + patch. */
int fk_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FK_H */
