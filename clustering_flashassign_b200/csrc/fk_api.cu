// The extern "C" surface of libfk (declared in include/fk.h): argument checks,
// dispatch to the kernels, the Lloyd loop and its streamed (out-of-core) path.
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "fk_internal.h"

namespace fk {

int check_shape(int B, long long N, int K, int d, int dtype) {
  if (dtype != FK_F32 && dtype != FK_F16 && dtype != FK_BF16)
    return set_error(FK_EINVAL, "unknown dtype " + std::to_string(dtype));
  if (B <= 0 || N <= 0 || K <= 0 || d <= 0) return set_error(FK_EINVAL, "B, N, K and d must be positive");
  if (N > 0x7fffffffLL) return set_error(FK_EINVAL, "N must be below 2^31");
  if ((long long)K > N) return set_error(FK_EINVAL, "K must not exceed N");
  if (B > 65535) return set_error(FK_EUNSUPPORTED, "B above 65535");
  if (K > (1 << 24)) return set_error(FK_EUNSUPPORTED, "K above 2^24");
  if (dtype != FK_F32 && (d * 2) % 16 != 0)
    return set_error(FK_EINVAL, "fp16/bf16 rows must be a multiple of 16 bytes (d % 8 == 0)");
  return FK_OK;
}

namespace {

enum Loc { LOC_DEVICE, LOC_HOST_PINNED, LOC_HOST_PAGEABLE };

Loc locate(const void *p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return LOC_HOST_PAGEABLE;
  }
  if (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) return LOC_DEVICE;
  if (at.type == cudaMemoryTypeHost) return LOC_HOST_PINNED;
  return LOC_HOST_PAGEABLE;
}

// Options with the environment's defaults: FK_VERBOSE=1 turns the per-iteration
// line on, FK_CHUNK_POINTS sets the streamed chunk size when the caller left it 0.
fk_options options_of(const fk_options *opts) {
  fk_options o{FK_HOST_AUTO, 0, 0};
  if (opts) o = *opts;
  if (const char *e = getenv("FK_VERBOSE"))
    if (atoi(e) != 0) o.verbose = 1;
  if (o.chunk_points <= 0)
    if (const char *e = getenv("FK_CHUNK_POINTS")) o.chunk_points = atoll(e);
  return o;
}

int check_ptr(const void *p, const char *name, bool aligned16) {
  if (!p) return set_error(FK_EINVAL, std::string(name) + " is NULL");
  if (aligned16 && (reinterpret_cast<uintptr_t>(p) & 15u))
    return set_error(FK_EINVAL, std::string(name) + " is not 16-byte aligned");
  return FK_OK;
}

// A pointer that the current device's kernels read or write: memory of this
// device, or managed memory.  Host memory and another device's memory are
// refused here instead of reaching a kernel.
int check_dev(const void *p, const char *name) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return set_error(FK_EINVAL, std::string(name) + " must be device memory");
  }
  if (at.type == cudaMemoryTypeManaged) return FK_OK;
  if (at.type != cudaMemoryTypeDevice) return set_error(FK_EINVAL, std::string(name) + " must be device memory");
  int dev = 0;
  FK_CUDA(cudaGetDevice(&dev));
  if (at.device != dev)
    return set_error(FK_EINVAL, std::string(name) + " is memory of device " + std::to_string(at.device) +
                                    ", not of the current device " + std::to_string(dev));
  return FK_OK;
}

int check_dev_opt(const void *p, const char *name) { return p ? check_dev(p, name) : FK_OK; }

// An argument that may be host or device memory: device memory must be this device's.
int check_if_dev(const void *p, Loc where, const char *name) {
  return where == LOC_DEVICE ? check_dev(p, name) : FK_OK;
}

int read_device_error(Workspace *ws, cudaStream_t s) {
  int h = 0;
  FK_CUDA(cudaMemcpyAsync(&h, ws->err, sizeof(int), cudaMemcpyDeviceToHost, s));
  FK_CUDA(cudaStreamSynchronize(s));
  if (h == DEV_OK) return FK_OK;
  FK_CUDA(cudaMemsetAsync(ws->err, 0, sizeof(int), s));
  FK_CUDA(cudaStreamSynchronize(s));
  if (h == DEV_TIMEOUT) return set_error(FK_ETIMEOUT, "a kernel's bounded wait expired");
  if (h == DEV_RANGE)
    return set_error(FK_EUNSUPPORTED,
                     "a squared norm reached 2^32, beyond the fp16 tensor-core norm digits");
  return set_error(FK_EINVAL, "an id outside [0, K) reached the update");
}

// Scratch of one update over B batches of n sorted positions: sorted
// (id, point) pairs, segment offsets, owner partial sums (B, K, d) and continuation
// partials (B, pieces, d).  Nothing here needs clearing: every value read is
// written by the same update first.
int prepare_update(Workspace *ws, int B, long long n, int K, int d) {
  FK_TRY(ensure(ws->kv, (size_t)B * n * sizeof(int2)));
  FK_TRY(ensure(ws->offsets, (size_t)B * K * sizeof(int32_t)));
  FK_TRY(ensure(ws->sums, (size_t)B * K * d * sizeof(float)));
  FK_TRY(ensure(ws->first, (size_t)B * pieces_of(n) * d * sizeof(float)));
  return FK_OK;
}

// Steps a2-a5 on device-resident points; ch / cnx (nullable) receive the dtype
// copy and the tensor-core extension rows of the new centroids for the next assign.
// have_hist: ws->table already holds the sort's tile histogram (accumulated by
// the assign), so the sort skips its histogram kernel.
int do_update(Workspace *ws, const void *x, const int32_t *ids, int B, long long N, int K, int d,
              int dtype, float *centers, int32_t *counts_out, void *ch, void *cnx, long long Kpad,
              cudaStream_t s, bool have_hist = false) {
  note_update_call();
  PhaseTimer whole(PH_UPDATE, s);
  int32_t *counts = counts_out;
  if (!counts) {
    FK_TRY(ensure(ws->counts, (size_t)B * K * sizeof(int32_t)));
    counts = (int32_t *)ws->counts.p;
  }
  FK_TRY(prepare_update(ws, B, N, K, d));
  // the max-shift word is zeroed by the sort's scan kernel (no memset between
  // the dependent launches of the update)
  int2 *kv = (int2 *)ws->kv.p;
  int32_t *offsets = (int32_t *)ws->offsets.p;
  float *sums = (float *)ws->sums.p, *first = (float *)ws->first.p;
  {
    PhaseTimer t(PH_SORT, s);
    if (have_hist) FK_TRY(run_sort_prehist(ws, ids, B, N, K, counts, offsets, nullptr, kv, s));
    else FK_TRY(run_sort(ws, ids, B, N, K, counts, offsets, nullptr, kv, s));
  }
  {
    PhaseTimer t(PH_REDUCE, s);
    FK_TRY(launch_segreduce(x, dtype, kv, B, N, K, d, sums, first, s));
  }
  PhaseTimer t(PH_FINALIZE, s);
  return launch_finalize(sums, first, pieces_of(N), counts, offsets, centers, ch, cnx, dtype, B, K,
                         d, Kpad, ws->maxshift, true, ws->err, s);
}

// fp32 on the tensor cores: the centroids' [hi | lo | hi] rows and tf32 norm
// rows every call; the points' [hi | hi | lo] rows from x3 when the caller
// prepared them (a Lloyd run does it once), else built here.
int assign_f32_tc(Workspace *ws, const float *x, const float *c, const float *x3, int B, long long N,
                  int K, int d, long long Kpad, int32_t *ids, cudaStream_t s, uint32_t *hist) {
  const int d3 = 3 * d;
  if (!x3) {
    FK_TRY(ensure(ws->x3, (size_t)B * N * d3 * sizeof(float)));
    FK_TRY(launch_split3(x, (long long)B * N, d, (float *)ws->x3.p, false, s));
    x3 = (const float *)ws->x3.p;
  }
  FK_TRY(ensure(ws->c3, (size_t)B * K * d3 * sizeof(float)));
  FK_TRY(launch_split3(c, (long long)B * K, d, (float *)ws->c3.p, true, s));
  FK_TRY(ensure(ws->cn, ext_bytes(B, Kpad)));
  FK_TRY(launch_prep_ext_f32(c, B, K, d, Kpad, ws->cn.p, s));
  // the widened point tiles (128 x 3d x 4 bytes) do not stay in L2 across a
  // tile's chunks: one work item per (tile, chunk), consecutive CTAs sharing a
  // tile's reads, merged through per-point keys
  FK_TRY(ensure_zeroed(ws->keys64, (size_t)B * N * sizeof(unsigned long long), s));
  // the keys are cleared by the kernel that turns them into ids; if an earlier
  // call stopped between the two launches they are cleared here
  if (ws->keys_dirty) FK_CUDA(cudaMemsetAsync(ws->keys64.p, 0, ws->keys64.bytes, s));
  ws->keys_dirty = true;
  FK_TRY(launch_assign_tc(x3, ws->c3.p, ws->cn.p, nullptr, FK_F32, B, N, K, d3, Kpad, ids, ws->err, s,
                          hist, (unsigned long long *)ws->keys64.p));
  ws->keys_dirty = false;
  return FK_OK;
}

int do_assign_resident(Workspace *ws, const void *x, const void *cdt, const void *cnx,
                       const float *xn, int B, long long N, int K, int d, int dtype, long long Kpad,
                       int32_t *ids, cudaStream_t s, uint32_t *hist = nullptr,
                       const float *x3 = nullptr, float *xn_out = nullptr) {
  PhaseTimer t(PH_ASSIGN, s);
  if (dtype == FK_F32) {
    if (use_tf32(K, d))
      return assign_f32_tc(ws, (const float *)x, (const float *)cdt, x3, B, N, K, d, Kpad, ids, s, hist);
    return launch_assign_f32((const float *)x, (const float *)cdt, B, N, K, d, ids, s);
  }
  // 16-bit split-d tiles (128 x d x 2 bytes) stay in L2 across a tile's
  // chunks, so one work item per tile (no per-chunk merge) is the faster order
  return launch_assign_tc(x, cdt, cnx, xn, dtype, B, N, K, d, Kpad, ids, ws->err, s, hist, nullptr, xn_out);
}

int read_shift(Workspace *ws, cudaStream_t s, float *out) {
  FK_CUDA(cudaMemcpyAsync(ws->h_maxshift, ws->maxshift, sizeof(float), cudaMemcpyDeviceToHost, s));
  FK_CUDA(cudaStreamSynchronize(s));
  *out = *ws->h_maxshift;
  return FK_OK;
}

int ensure_copy_engine(Workspace *ws) {
  if (!ws->copy_stream) FK_CUDA(cudaStreamCreateWithFlags(&ws->copy_stream, cudaStreamNonBlocking));
  for (int i = 0; i < 2; ++i) {
    if (!ws->ready[i]) FK_CUDA(cudaEventCreateWithFlags(&ws->ready[i], cudaEventDisableTiming));
    if (!ws->freed[i]) FK_CUDA(cudaEventCreateWithFlags(&ws->freed[i], cudaEventDisableTiming));
  }
  return FK_OK;
}

// Scratch of the streamed pipeline: the copy stream and events, two chunk
// buffers, and the per-chunk update scratch (one batch of `chunk` points).
int prepare_streamed(Workspace *ws, const fk_shape &sh, long long chunk) {
  FK_TRY(ensure_copy_engine(ws));
  for (int i = 0; i < 2; ++i) FK_TRY(ensure(ws->chunk[i], (size_t)chunk * sh.d * esize(sh.dtype)));
  FK_TRY(ensure(ws->counts, (size_t)sh.K * sizeof(int32_t)));
  return prepare_update(ws, 1, chunk, sh.K, sh.d);
}

// One pass of the out-of-core pipeline over every batch: x stays in host
// memory and is streamed in chunks, double-buffered so the copy of chunk j+1
// overlaps the compute of chunk j ("flash-kmeans and the return of exact
// K-Means on the GPU", section "Multi-GPU scaling without a NCCL dependency":
// per-device double-buffered host-to-device plus compute pipeline).  Each
// chunk is assigned against `cassign` (B, K, d) in x's dtype, sorted and
// segment-reduced, and its sums and counts are folded into gsum / gcounts
// (zeroed first).  ws->stream_job numbers the chunks across passes, so the
// two buffers keep alternating and the next pass's first copy can start while
// the current pass is still being reduced.
int streamed_pass(Workspace *ws, const fk_shape &sh, const char *xh, long long chunk,
                  const void *cassign, const char *cnx, int32_t *ids_dev, float *gsum,
                  int32_t *gcounts, cudaStream_t s) {
  const int B = sh.B, K = sh.K, d = sh.d, dtype = sh.dtype;
  const long long N = sh.N;
  const size_t es = esize(dtype);
  const long long Kpad = kpad_of(K);
  const long long per_b = (N + chunk - 1) / chunk;
  int32_t *counts = (int32_t *)ws->counts.p;
  float *sums = (float *)ws->sums.p, *first = (float *)ws->first.p;
  int2 *kv = (int2 *)ws->kv.p;
  int32_t *offsets = (int32_t *)ws->offsets.p;
  note_update_call();
  FK_CUDA(cudaMemsetAsync(gcounts, 0, (size_t)B * K * sizeof(int32_t), s));
  FK_CUDA(cudaMemsetAsync(gsum, 0, (size_t)B * K * d * sizeof(float), s));
  for (int b = 0; b < B; ++b) {
    for (long long ci = 0; ci < per_b; ++ci, ++ws->stream_job) {
      const int buf = (int)(ws->stream_job & 1);
      const long long n0 = ci * chunk;
      const long long nc = (n0 + chunk <= N) ? chunk : N - n0;
      void *xb = ws->chunk[buf].p;
      FK_CUDA(cudaStreamWaitEvent(ws->copy_stream, ws->freed[buf], 0));
      if (fault_hit(FK_FAULT_H2D)) return set_error(FK_ECUDA, "injected host-to-device copy failure (FK_FAULT)");
      FK_TRY(chunk_event(0, ws->stream_job, buf, ws->copy_stream));
      FK_CUDA(cudaMemcpyAsync(xb, xh + ((size_t)b * N + n0) * d * es, (size_t)nc * d * es,
                              cudaMemcpyHostToDevice, ws->copy_stream));
      FK_TRY(chunk_event(1, ws->stream_job, buf, ws->copy_stream));
      FK_CUDA(cudaEventRecord(ws->ready[buf], ws->copy_stream));
      FK_CUDA(cudaStreamWaitEvent(s, ws->ready[buf], 0));
      FK_TRY(chunk_event(2, ws->stream_job, buf, s));
      int32_t *idc = ids_dev + (size_t)b * N + n0;
      const void *cb = (const char *)cassign + (size_t)b * K * d * es;
      FK_TRY(do_assign_resident(ws, xb, cb, cnx ? cnx + ext_bytes(b, Kpad) : nullptr, nullptr, 1, nc, K,
                                d, dtype, Kpad, idc, s));
      {
        PhaseTimer t(PH_SORT, s);
        FK_TRY(run_sort(ws, idc, 1, nc, K, counts, offsets, nullptr, kv, s));
      }
      {
        PhaseTimer t(PH_REDUCE, s);
        FK_TRY(launch_segreduce(xb, dtype, kv, 1, nc, K, d, sums, first, s));
        FK_TRY(launch_accumulate(sums, first, pieces_of(nc), counts, offsets, 1, K, d,
                                 gsum + (size_t)b * K * d, gcounts + (size_t)b * K, false, s));
      }
      FK_TRY(chunk_event(3, ws->stream_job, buf, s));
      FK_CUDA(cudaEventRecord(ws->freed[buf], s));
    }
  }
  return FK_OK;
}

// Out-of-core Lloyd: one streamed pass per iteration (assign, sort and
// segment reduce per chunk), then one finalize per iteration.
int lloyd_streamed(Workspace *ws, const fk_shape &sh, const char *xh, const void *init_dev,
                   int max_iter, float tol, int32_t *ids_dev, float *cen_dev, cudaStream_t s,
                   int *iters_run, long long chunk, int verbose) {
  const int B = sh.B, K = sh.K, d = sh.d, dtype = sh.dtype;
  const size_t es = esize(dtype);
  const long long Kpad = kpad_of(K);
  if (chunk <= 0) chunk = 1LL << 24;
  if (chunk > sh.N) chunk = sh.N;
  FK_TRY(prepare_streamed(ws, sh, chunk));
  void *ch = nullptr;
  char *cnx = nullptr;
  if (dtype != FK_F32) {
    FK_TRY(ensure(ws->ch, (size_t)B * K * d * es));
    FK_TRY(ensure(ws->cn, ext_bytes(B, Kpad)));
    ch = ws->ch.p;
    cnx = (char *)ws->cn.p;
  }
  // per iteration: running sums and counts of every batch
  FK_TRY(ensure(ws->gsum, (size_t)B * K * d * sizeof(float)));
  FK_TRY(ensure(ws->gcounts, (size_t)B * K * sizeof(int32_t)));
  int32_t *gcounts = (int32_t *)ws->gcounts.p;
  float *gsum = (float *)ws->gsum.p;
  FK_TRY(launch_init_centers(init_dev, dtype, B, K, d, Kpad, cen_dev, ch, cnx, ws->err, s));
  const void *cassign = dtype == FK_F32 ? (const void *)cen_dev : ch;
  int it = 0;
  for (it = 0; it < max_iter; ++it) {
    FK_CUDA(cudaMemsetAsync(ws->maxshift, 0, sizeof(unsigned), s));
    FK_TRY(streamed_pass(ws, sh, xh, chunk, cassign, cnx, ids_dev, gsum, gcounts, s));
    {
      PhaseTimer t(PH_FINALIZE, s);
      FK_TRY(launch_finalize(gsum, nullptr, 0, gcounts, nullptr, cen_dev, ch, cnx, dtype, B, K, d,
                             Kpad, ws->maxshift, false, ws->err, s));
    }
    if (tol > 0.f || verbose) {
      float ms = 0.f;
      FK_TRY(read_shift(ws, s, &ms));
      if (verbose) fprintf(stderr, "fk_lloyd(streamed) iter %d max_shift %.6g\n", it + 1, ms);
      if (tol > 0.f && ms < tol) {
        ++it;
        break;
      }
    }
  }
  *iters_run = it;
  return FK_OK;
}

// Steps a2-a5 without the division, on device-resident points: the
// per-cluster sums (B, K, d) fp32 and counts (B, K) of these points, written
// to the caller's buffers (an empty cluster gets zeros).  have_hist as in
// do_update.
int do_partial(Workspace *ws, const void *x, const int32_t *ids, int B, long long N, int K, int d,
               int dtype, float *sums_out, int32_t *counts_out, cudaStream_t s, bool have_hist) {
  note_update_call();
  PhaseTimer whole(PH_UPDATE, s);
  FK_TRY(prepare_update(ws, B, N, K, d));
  int2 *kv = (int2 *)ws->kv.p;
  int32_t *offsets = (int32_t *)ws->offsets.p;
  float *sums = (float *)ws->sums.p, *first = (float *)ws->first.p;
  {
    PhaseTimer t(PH_SORT, s);
    if (have_hist) FK_TRY(run_sort_prehist(ws, ids, B, N, K, counts_out, offsets, nullptr, kv, s));
    else FK_TRY(run_sort(ws, ids, B, N, K, counts_out, offsets, nullptr, kv, s));
  }
  {
    PhaseTimer t(PH_REDUCE, s);
    FK_TRY(launch_segreduce(x, dtype, kv, B, N, K, d, sums, first, s));
  }
  PhaseTimer t(PH_FINALIZE, s);
  return launch_accumulate(sums, first, pieces_of(N), counts_out, offsets, B, K, d, sums_out, nullptr,
                           true, s);
}

}  // namespace
}  // namespace fk

using namespace fk;

extern "C" {

int fk_assign(const void *x, const void *c, int B, long long N, int K, int d, int dtype,
              int32_t *ids, fk_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  FK_TRY(check_shape(B, N, K, d, dtype));
  const bool tc = dtype != FK_F32;
  FK_TRY(check_ptr(x, "x", tc));
  FK_TRY(check_ptr(c, "c", tc));
  FK_TRY(check_ptr(ids, "ids", false));
  FK_TRY(check_dev(x, "x"));
  FK_TRY(check_dev(c, "c"));
  FK_TRY(check_dev(ids, "ids"));
  Workspace *ws;
  FK_TRY(workspace_for(s, &ws));
  const long long Kpad = kpad_of(K);
  void *cnx = nullptr;
  if (tc) {
    FK_TRY(ensure(ws->cn, ext_bytes(B, Kpad)));
    cnx = ws->cn.p;
    FK_TRY(launch_prep_cn(c, dtype, B, K, d, Kpad, cnx, ws->err, s));
  }
  return do_assign_resident(ws, x, c, cnx, nullptr, B, N, K, d, dtype, Kpad, ids, s);
}

int fk_update(const void *x, const int32_t *ids, int B, long long N, int K, int d, float *centers,
              int32_t *counts, fk_stream_t stream, int dtype, float *max_shift) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  FK_TRY(check_shape(B, N, K, d, dtype));
  FK_TRY(check_ptr(x, "x", true));
  FK_TRY(check_ptr(ids, "ids", false));
  FK_TRY(check_ptr(centers, "centers", true));
  FK_TRY(check_dev(x, "x"));
  FK_TRY(check_dev(ids, "ids"));
  FK_TRY(check_dev(centers, "centers"));
  FK_TRY(check_dev_opt(counts, "counts"));
  FK_TRY(check_dev_opt(max_shift, "max_shift"));
  Workspace *ws;
  FK_TRY(workspace_for(s, &ws));
  FK_TRY(do_update(ws, x, ids, B, N, K, d, dtype, centers, counts, nullptr, nullptr, kpad_of(K), s));
  if (max_shift)
    FK_CUDA(cudaMemcpyAsync(max_shift, ws->maxshift, sizeof(float), cudaMemcpyDeviceToDevice, s));
  return FK_OK;
}

int fk_sort(const int32_t *ids, int B, long long N, int K, int32_t *counts, int32_t *offsets,
            int32_t *perm, fk_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  FK_TRY(check_shape(B, N, K, 8, FK_F32));
  FK_TRY(check_ptr(ids, "ids", false));
  FK_TRY(check_ptr(perm, "perm", false));
  FK_TRY(check_dev(ids, "ids"));
  FK_TRY(check_dev(perm, "perm"));
  FK_TRY(check_dev_opt(counts, "counts"));
  FK_TRY(check_dev_opt(offsets, "offsets"));
  Workspace *ws;
  FK_TRY(workspace_for(s, &ws));
  PhaseTimer t(PH_SORT, s);
  return run_sort(ws, ids, B, N, K, counts, offsets, perm, nullptr, s);
}

int fk_point_norms(const void *x, int B, long long N, int d, int dtype, float *xn,
                   fk_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  FK_TRY(check_shape(B, N, 1, d, dtype));
  if (dtype == FK_F32) return set_error(FK_EUNSUPPORTED, "point norms serve the fp16 / bf16 assign");
  FK_TRY(check_ptr(x, "x", true));
  FK_TRY(check_ptr(xn, "xn", false));
  FK_TRY(check_dev(x, "x"));
  FK_TRY(check_dev(xn, "xn"));
  return launch_point_norms(x, dtype, (long long)B * N, d, xn, s);
}

int fk_init_centers(const void *init, int B, int K, int d, int dtype, float *centers,
                    fk_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  FK_TRY(check_shape(B, K, K, d, dtype));
  FK_TRY(check_ptr(init, "init", false));
  FK_TRY(check_ptr(centers, "centers", false));
  FK_TRY(check_dev(init, "init"));
  FK_TRY(check_dev(centers, "centers"));
  Workspace *ws;
  FK_TRY(workspace_for(s, &ws));
  return launch_init_centers(init, dtype, B, K, d, kpad_of(K), centers, nullptr, nullptr, ws->err, s);
}

int fk_lloyd_step_partial(const fk_shape *shape, const void *x, const float *xn,
                          const void *centers_dt, int32_t *ids, float *sums, int32_t *counts,
                          fk_stream_t stream, const fk_options *opts) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!shape) return set_error(FK_EINVAL, "shape is NULL");
  const fk_shape sh = *shape;
  const int B = sh.B, K = sh.K, d = sh.d, dtype = sh.dtype;
  const long long N = sh.N;
  // a rank's block of a larger problem may hold fewer points than there are
  // clusters, or none: only the whole problem needs K <= N
  if (N < 0) return set_error(FK_EINVAL, "N must be >= 0");
  FK_TRY(check_shape(B, N > K ? N : K, K, d, dtype));
  const bool tc = dtype != FK_F32;
  if (N > 0) {
    FK_TRY(check_ptr(x, "x", tc));
    FK_TRY(check_ptr(ids, "ids", false));
  }
  FK_TRY(check_ptr(centers_dt, "centers_dt", tc));
  FK_TRY(check_ptr(sums, "sums", false));
  FK_TRY(check_ptr(counts, "counts", false));
  FK_TRY(check_dev(centers_dt, "centers_dt"));
  FK_TRY(check_dev(sums, "sums"));
  FK_TRY(check_dev(counts, "counts"));
  if (N == 0) {  // an empty block contributes nothing to the totals
    FK_CUDA(cudaMemsetAsync(sums, 0, (size_t)B * K * d * sizeof(float), s));
    FK_CUDA(cudaMemsetAsync(counts, 0, (size_t)B * K * sizeof(int32_t), s));
    return FK_OK;
  }
  FK_TRY(check_dev(ids, "ids"));
  FK_TRY(check_dev_opt(xn, "xn"));
  const fk_options o = options_of(opts);
  Workspace *ws;
  FK_TRY(workspace_for(s, &ws));
  const long long Kpad = kpad_of(K);
  char *cnx = nullptr;
  if (tc) {
    FK_TRY(ensure(ws->cn, ext_bytes(B, Kpad)));
    cnx = (char *)ws->cn.p;
    FK_TRY(launch_prep_cn(centers_dt, dtype, B, K, d, Kpad, cnx, ws->err, s));
  }
  const Loc lx = locate(x);
  if (lx == LOC_HOST_PAGEABLE) return set_error(FK_EINVAL, "x must be device or pinned host memory");
  FK_TRY(check_if_dev(x, lx, "x"));
  if (lx == LOC_HOST_PINNED) {
    long long chunk = o.chunk_points > 0 ? o.chunk_points : (1LL << 24);
    if (chunk > N) chunk = N;
    FK_TRY(prepare_streamed(ws, sh, chunk));
    return streamed_pass(ws, sh, (const char *)x, chunk, centers_dt, cnx, ids, sums, counts, s);
  }
  // With K <= 4096 the assign counts every id into the sort's tile histogram.
  const bool fuse = (tc || use_tf32(K, d)) && sort_single_pass(K);
  uint32_t *hist = nullptr;
  if (fuse) {
    const size_t hist_bytes = sort_table_bytes(B, N, K);
    FK_TRY(ensure(ws->table, hist_bytes));
    hist = (uint32_t *)ws->table.p;
    FK_CUDA(cudaMemsetAsync(hist, 0, hist_bytes, s));
  }
  // the resident assign ranks with the norms; the split-d one reads them for
  // its far-point check
  const float *xnr = tc ? xn : nullptr;
  FK_TRY(do_assign_resident(ws, x, centers_dt, cnx, xnr, B, N, K, d, dtype, Kpad, ids, s, hist));
  return do_partial(ws, x, ids, B, N, K, d, dtype, sums, counts, s, fuse);
}

int fk_update_finalize(const float *sums, const int32_t *counts, int B, int K, int d, int dtype,
                       float *centers, void *centers_dt, float *max_shift, fk_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  FK_TRY(check_shape(B, K, K, d, dtype));
  FK_TRY(check_ptr(sums, "sums", false));
  FK_TRY(check_ptr(counts, "counts", false));
  FK_TRY(check_ptr(centers, "centers", true));
  FK_TRY(check_dev(sums, "sums"));
  FK_TRY(check_dev(counts, "counts"));
  FK_TRY(check_dev(centers, "centers"));
  if (dtype != FK_F32) FK_TRY(check_dev_opt(centers_dt, "centers_dt"));
  FK_TRY(check_dev_opt(max_shift, "max_shift"));
  Workspace *ws;
  FK_TRY(workspace_for(s, &ws));
  FK_CUDA(cudaMemsetAsync(ws->maxshift, 0, sizeof(unsigned), s));
  {
    PhaseTimer t(PH_FINALIZE, s);
    FK_TRY(launch_finalize(sums, nullptr, 0, counts, nullptr, centers, dtype == FK_F32 ? nullptr : centers_dt,
                           nullptr, dtype, B, K, d, kpad_of(K), ws->maxshift, false, ws->err, s));
  }
  if (max_shift)
    FK_CUDA(cudaMemcpyAsync(max_shift, ws->maxshift, sizeof(float), cudaMemcpyDeviceToDevice, s));
  return FK_OK;
}

int fk_lloyd(const fk_shape *shape, const void *x, const void *init_centers, int max_iter,
             float tol, int32_t *ids, float *centers, fk_stream_t stream, int *iters_run,
             const fk_options *opts) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!shape) return set_error(FK_EINVAL, "shape is NULL");
  const fk_shape sh = *shape;
  FK_TRY(check_shape(sh.B, sh.N, sh.K, sh.d, sh.dtype));
  FK_TRY(check_ptr(x, "x", true));
  FK_TRY(check_ptr(init_centers, "init_centers", false));
  FK_TRY(check_ptr(ids, "ids", false));
  FK_TRY(check_ptr(centers, "centers", true));
  if (max_iter < 0) return set_error(FK_EINVAL, "max_iter must be >= 0");
  const fk_options o = options_of(opts);
  const int B = sh.B, K = sh.K, d = sh.d, dtype = sh.dtype;
  const long long N = sh.N;
  const size_t es = esize(dtype);
  const size_t xbytes = (size_t)B * N * d * es;
  const size_t cbytes = (size_t)B * K * d * es;
  const long long Kpad = kpad_of(K);
  Workspace *ws;
  FK_TRY(workspace_for(s, &ws));

  const Loc lx = locate(x), li = locate(init_centers), lids = locate(ids), lc = locate(centers);
  FK_TRY(check_if_dev(x, lx, "x"));
  FK_TRY(check_if_dev(init_centers, li, "init_centers"));
  FK_TRY(check_if_dev(ids, lids, "ids"));
  FK_TRY(check_if_dev(centers, lc, "centers"));
  const void *init_dev = init_centers;
  if (li != LOC_DEVICE) {
    FK_TRY(ensure(ws->init_dev, cbytes));
    if (fault_hit(FK_FAULT_H2D)) return set_error(FK_ECUDA, "injected host-to-device copy failure (FK_FAULT)");
    FK_CUDA(cudaMemcpyAsync(ws->init_dev.p, init_centers, cbytes, cudaMemcpyHostToDevice, s));
    init_dev = ws->init_dev.p;
  }
  int32_t *ids_dev = ids;
  if (lids != LOC_DEVICE) {
    FK_TRY(ensure(ws->ids_dev, (size_t)B * N * sizeof(int32_t)));
    ids_dev = (int32_t *)ws->ids_dev.p;
  }
  float *cen_dev = centers;
  if (lc != LOC_DEVICE) {
    FK_TRY(ensure(ws->centers_dev, (size_t)B * K * d * sizeof(float)));
    cen_dev = (float *)ws->centers_dev.p;
  }

  int iters = 0;
  bool streamed = false;
  const void *xdev = x;
  if (lx != LOC_DEVICE) {
    int mode = o.host_mode;
    if (mode == FK_HOST_AUTO) {
      size_t fr = 0, tot = 0;
      FK_CUDA(cudaMemGetInfo(&fr, &tot));
      mode = (xbytes + (size_t)(2ull << 30) < fr) ? FK_HOST_RESIDENT : FK_HOST_STREAM;
    }
    if (mode == FK_HOST_STREAM) {
      streamed = true;
      FK_TRY(lloyd_streamed(ws, sh, (const char *)x, init_dev, max_iter, tol, ids_dev, cen_dev, s,
                            &iters, o.chunk_points, o.verbose));
    } else {
      FK_TRY(ensure(ws->xres, xbytes));
      if (fault_hit(FK_FAULT_H2D)) return set_error(FK_ECUDA, "injected host-to-device copy failure (FK_FAULT)");
      FK_CUDA(cudaMemcpyAsync(ws->xres.p, x, xbytes, cudaMemcpyHostToDevice, s));
      xdev = ws->xres.p;
    }
  }
  if (!streamed) {
    void *ch = nullptr;
    void *cnx = nullptr;
    float *xn = nullptr;
    if (dtype != FK_F32) {
      FK_TRY(ensure(ws->ch, cbytes));
      FK_TRY(ensure(ws->cn, ext_bytes(B, Kpad)));
      ch = ws->ch.p;
      cnx = ws->cn.p;
      if (max_iter > 1 && d <= 2 * kBlockK) {
        // the resident-tile assign ranks with ||x||^2 too; the points do not
        // change, so the first assign stores the norms it computes from its
        // shared tiles and the later ones read them
        FK_TRY(ensure(ws->xn, (size_t)B * N * sizeof(float)));
        xn = (float *)ws->xn.p;
      } else if (max_iter > 0 && d > 2 * kBlockK) {
        // the split-d assign's far-point check reads ||x||^2: one pass over
        // the points per call instead of row reads in every assign
        FK_TRY(ensure(ws->xn, (size_t)B * N * sizeof(float)));
        xn = (float *)ws->xn.p;
        FK_TRY(launch_point_norms(xdev, dtype, (long long)B * N, d, xn, s));
      }
    }
    FK_TRY(launch_init_centers(init_dev, dtype, B, K, d, Kpad, cen_dev, ch, cnx, ws->err, s));
    const void *cassign = dtype == FK_F32 ? (const void *)cen_dev : ch;
    // The assign of iteration it+1 is queued before the host looks at the
    // shift of iteration it, so the GPU never idles during the tol check.  It
    // writes the other of two id buffers: when the check stops the loop, the
    // returned ids are still those of the last assign whose update produced
    // the returned centroids, and the queued assign is discarded.
    const bool check = tol > 0.f || o.verbose;
    int32_t *idbuf[2] = {ids_dev, ids_dev};
    if (check && max_iter > 1) {
      FK_TRY(ensure(ws->ids_alt, (size_t)B * N * sizeof(int32_t)));
      idbuf[1] = (int32_t *)ws->ids_alt.p;
      if (!ws->shift_ev) FK_CUDA(cudaEventCreateWithFlags(&ws->shift_ev, cudaEventDisableTiming));
    }
    // fp32 on the tensor cores: the points' [hi | hi | lo] rows once per call
    const bool tc32 = dtype == FK_F32 && use_tf32(K, d);
    const float *x3 = nullptr;
    if (tc32) {
      FK_TRY(ensure(ws->x3, (size_t)B * N * 3 * d * sizeof(float)));
      FK_TRY(launch_split3((const float *)xdev, (long long)B * N, d, (float *)ws->x3.p, false, s));
      x3 = (const float *)ws->x3.p;
    }
    // With K <= 4096 the tensor-core assign also counts every id into the
    // sort's tile histogram, so the sort starts at its scan.
    const bool fuse = (dtype != FK_F32 || tc32) && sort_single_pass(K);
    uint32_t *hist = nullptr;
    const size_t hist_bytes = sort_table_bytes(B, N, K);
    if (fuse) {
      FK_TRY(ensure(ws->table, hist_bytes));
      hist = (uint32_t *)ws->table.p;
    }
    // the table starts at zero; afterwards every sort's scatter zeroes the
    // rows it has read, so no memset separates the iterations' launches
    if (hist) FK_CUDA(cudaMemsetAsync(hist, 0, hist_bytes, s));
    auto assign = [&](int32_t *out) -> int {
      return do_assign_resident(ws, xdev, cassign, cnx, xn, B, N, K, d, dtype, Kpad, out, s, hist, x3);
    };
    int cur = 0;
    if (max_iter > 0)  // resident: the first assign computes the point norms and keeps them in xn
      FK_TRY(do_assign_resident(ws, xdev, cassign, cnx, d > 2 * kBlockK ? xn : nullptr, B, N, K, d, dtype, Kpad,
                                idbuf[0], s, hist, x3, xn));
    for (int it = 0; it < max_iter; ++it) {
      FK_TRY(do_update(ws, xdev, idbuf[cur], B, N, K, d, dtype, cen_dev, nullptr, ch, cnx, Kpad, s, fuse));
      iters = it + 1;
      const bool last = it + 1 == max_iter;
      if (check) {
        FK_CUDA(cudaMemcpyAsync(ws->h_maxshift, ws->maxshift, sizeof(float), cudaMemcpyDeviceToHost, s));
        if (ws->shift_ev) FK_CUDA(cudaEventRecord(ws->shift_ev, s));
        if (!last) FK_TRY(assign(idbuf[cur ^ 1]));
        if (ws->shift_ev) FK_CUDA(cudaEventSynchronize(ws->shift_ev));
        else FK_CUDA(cudaStreamSynchronize(s));
        const float ms = *ws->h_maxshift;
        if (o.verbose) fprintf(stderr, "fk_lloyd iter %d max_shift %.6g\n", it + 1, ms);
        if (tol > 0.f && ms < tol) break;
        if (!last) cur ^= 1;
      } else if (!last) {
        FK_TRY(assign(idbuf[0]));
      }
    }
    if (idbuf[cur] != ids_dev)
      FK_CUDA(cudaMemcpyAsync(ids_dev, idbuf[cur], (size_t)B * N * sizeof(int32_t), cudaMemcpyDeviceToDevice, s));
  }
  if (ids_dev != ids)
    FK_CUDA(cudaMemcpyAsync(ids, ids_dev, (size_t)B * N * sizeof(int32_t), cudaMemcpyDeviceToHost, s));
  if (cen_dev != centers)
    FK_CUDA(cudaMemcpyAsync(centers, cen_dev, (size_t)B * K * d * sizeof(float), cudaMemcpyDeviceToHost, s));
  FK_CUDA(cudaStreamSynchronize(s));
  FK_TRY(read_device_error(ws, s));
  if (iters_run) *iters_run = iters;
  return FK_OK;
}

const char *fk_status_string(int status) {
  switch (status) {
    case FK_OK: return "ok";
    case FK_EINVAL: return "invalid argument";
    case FK_ENOMEM: return "out of device memory";
    case FK_ECUDA: return "CUDA runtime error";
    case FK_ETIMEOUT: return "kernel wait timed out";
    case FK_EUNSUPPORTED: return "unsupported shape";
    default: return "unknown status";
  }
}

const char *fk_last_error(void) { return last_error(); }

int fk_device_error(fk_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Workspace *ws;
  FK_TRY(workspace_for(s, &ws));
  return read_device_error(ws, s);
}

int fk_release(void) {
  FK_CUDA(cudaDeviceSynchronize());
  return release_device_workspaces();
}

int fk_profile_enable(int on) { return profile_enable(on); }

int fk_profile_read(fk_profile *out, int reset) { return profile_read(out, reset); }

int fk_profile_timeline(double *out, int max_chunks, int *rows) {
  if (max_chunks < 0) return set_error(FK_EINVAL, "max_chunks must be >= 0");
  int n = 0;
  FK_TRY(profile_timeline(out, max_chunks, &n));
  if (rows) *rows = n;
  return FK_OK;
}

long long fk_launch_count(void) { return launch_count(); }

int fk_version(void) { return 100; }

int fk_inject_fault(int kind, long long nth) { return set_fault(kind, nth); }

}  // extern "C"
