// Internal declarations shared by the libfk CUDA sources.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <string>

#include "../../include/fk.h"

namespace fk {

// Device error word values (written by kernels, read by fk_device_error).
// DEV_RANGE: a squared norm beyond the range of the fp16 norm digits that
// the tensor-core assign folds into its MMA (||v||^2 >= 2^32).
enum : int { DEV_OK = 0, DEV_TIMEOUT = 1, DEV_BAD_ID = 2, DEV_RANGE = 3 };

// Bounded waits inside kernels give up after this many nanoseconds.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

// Tile geometry of the tensor-core assign.
constexpr int kTileM = 128;   // points per tile (MMA M)
constexpr int kChunkN = 256;  // centroids per chunk (MMA N)
constexpr int kBlockK = 64;   // elements of d per K-block (128-byte rows for 16-bit types)

inline long long kpad_of(int K) { return ((long long)K + kChunkN - 1) / kChunkN * kChunkN; }

// Bytes of the tensor-core extension rows of `B` batches: (B, Kpad, 16) 16-bit
// elements (the norm digits folded into the MMA, fk_norms.cuh).
constexpr int kExtElems = 16;
inline size_t ext_bytes(long long B, long long Kpad) { return (size_t)B * Kpad * kExtElems * 2; }

// Counting-sort geometry.
constexpr int kSortTile = 2048;    // points per sort tile (one warp walks it in order)
constexpr int kMaxDigitBits = 12;                         // 4096 bins per pass at most

// Segment-reduce geometry.
constexpr int kPiece = 128;  // sorted positions per segment piece

inline int pieces_of(long long N) { return (int)((N + kPiece - 1) / kPiece); }

struct DevBuf {
  void *p = nullptr;
  size_t bytes = 0;
};

// Per (device, stream) scratch.  Grow-only; freed by fk_release().
struct Workspace {
  int device = -1;
  cudaStream_t stream = nullptr;
  int *err = nullptr;             // device error word
  unsigned *maxshift = nullptr;   // device, float bits (non-negative floats order as uints)
  float *h_maxshift = nullptr;    // pinned host mirror
  DevBuf cn, ch, sums, first, counts, offsets, table, digit_off, kv, keys_b, vals_b;
  DevBuf xres, init_dev, ids_dev, centers_dev, chunk[2], gsum, gcounts, xn, ids_alt;
  DevBuf x3, c3;                  // 3xTF32 operands of the fp32 tensor-core assign
  DevBuf keys64;                  // split-d per-point argmax keys, kept zeroed
  bool keys_dirty = false;        // an assign wrote keys64 that nothing has cleared yet
  cudaStream_t copy_stream = nullptr;
  cudaEvent_t ready[2] = {nullptr, nullptr}, freed[2] = {nullptr, nullptr};
  cudaEvent_t shift_ev = nullptr;  // the max-shift copy of the Lloyd loop has landed
  long long stream_job = 0;        // chunks streamed so far (selects the chunk buffer)
};

// Status plumbing (thread-local last-error text).
int set_error(int status, const std::string &msg);
int cuda_status(cudaError_t e, const char *what);
#define FK_CUDA(call)                                        \
  do {                                                       \
    cudaError_t e_ = (call);                                 \
    if (e_ != cudaSuccess) return ::fk::cuda_status(e_, #call); \
  } while (0)
#define FK_TRY(expr)              \
  do {                            \
    int s_ = (expr);              \
    if (s_ != FK_OK) return s_;   \
  } while (0)

int ensure(DevBuf &b, size_t bytes);               // grow-only device buffer
int ensure_zeroed(DevBuf &b, size_t bytes, cudaStream_t s);  // zero-filled when (re)allocated
int workspace_for(cudaStream_t s, Workspace **out);
// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device, once per (device, kernel).
int set_smem_limit(const void *func, int bytes);

// Launch accounting and event timing.
// Launch accounting; returns FK_ECUDA when an injected launch fault fires.
int launched(int n = 1);
// Host-side fault injection: true when the armed failure of `kind`
// (FK_FAULT_ALLOC / _H2D / _LAUNCH) fires here.
bool fault_hit(int kind);
int set_fault(int kind, long long nth);
enum Phase { PH_ASSIGN = 0, PH_SORT = 1, PH_REDUCE = 2, PH_FINALIZE = 3, PH_UPDATE = 4, PH_COUNT = 5 };
struct PhaseTimer {
  cudaEvent_t a = nullptr, b = nullptr;
  int phase;
  cudaStream_t s;
  PhaseTimer(int ph, cudaStream_t st);
  ~PhaseTimer();
};
void note_update_call();
int release_device_workspaces();
long long launch_count();
int profile_enable(int on);
int profile_read(fk_profile *out, int reset);
// Level 3: per-chunk events of the streamed pipeline.  which: 0 copy begin,
// 1 copy end (on the copy stream), 2 compute begin, 3 compute end (on the
// compute stream); 0 opens the chunk's record.
bool timeline_on();
int chunk_event(int which, long long chunk, int buf, cudaStream_t s);
int profile_timeline(double *out, int max_chunks, int *rows);
const char *last_error();

size_t esize(int dtype);
int num_sms();

// Shape and dtype rules shared by every entry point that takes (B, N, K, d):
// FK_EINVAL for an unknown dtype, a size <= 0, N >= 2^31, K > N, or 16-bit
// rows that are not a multiple of 16 bytes; FK_EUNSUPPORTED for B > 65535 or
// K > 2^24.
int check_shape(int B, long long N, int K, int d, int dtype);

// Programmatic dependent launch: the kernels of one Lloyd iteration are
// launched so that each may start while its predecessor in the stream drains.
// A kernel launched this way calls pdl_wait() before it reads anything an
// earlier kernel of the stream writes (or writes anything an earlier kernel
// still reads), and pdl_trigger() only after its own pdl_wait(), so a kernel
// that has started implies that every kernel two or more launches back has
// completed.  After a memset or a copy the launch is ordinary.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ---- kernels (launchers return fk_status) ----
// Centroid preparation for the tensor-core assign: cnx[b, k, 0..15] = the
// extension row of centroid k (digits of ||c||^2 / 2, see fk_norms.cuh), zero
// rows on [K, Kpad).  Only for 16-bit dtypes (cnx is (B, Kpad, 16) in dtype).
int launch_prep_cn(const void *c, int dtype, int B, int K, int d, long long Kpad, void *cnx,
                   int *err, cudaStream_t s);
// init for fk_lloyd: master = float(init), ch = init and cnx (16-bit dtypes).
int launch_init_centers(const void *init, int dtype, int B, int K, int d, long long Kpad,
                        float *master, void *ch, void *cnx, int *err, cudaStream_t s);
// finalize: new = (segment sum) / count or old; max shift; master, ch, cnx.
// from_pieces: the segment sum is sums[k] plus the continuation partials of
// the following pieces (fk_reduce.cu); otherwise sums[k] is complete.
int launch_finalize(const float *sums, const float *first, int pieces, const int32_t *counts,
                    const int32_t *offsets, float *centers, void *ch, void *cnx, int dtype, int B,
                    int K, int d, long long Kpad, unsigned *maxshift, bool from_pieces, int *err,
                    cudaStream_t s);
// per-cluster totals of the segment partials of B batches: gsum[b][k] = the
// segment sum (overwrite) or gsum[b][k] += it and gcounts[b][k] += counts[b][k].
int launch_accumulate(const float *sums, const float *first, int pieces, const int32_t *counts,
                      const int32_t *offsets, int B, int K, int d, float *gsum, int32_t *gcounts,
                      bool overwrite, cudaStream_t s);

int launch_assign_f32(const float *x, const float *c, int B, long long N, int K, int d,
                      int32_t *ids, cudaStream_t s);
// fp32 on the tensor cores (3xTF32, fk_tf32.cu): used when d % 4 == 0 and
// K * d >= kTf32MinKd; smaller problems stay on the CUDA-core kernel.
constexpr long long kTf32MinKd = 16384;
bool use_tf32(int K, int d);
// dst (rows, 3d) = [hi | hi | lo] (points) or [hi | lo | hi] (centroids) of src (rows, d).
int launch_split3(const float *src, long long rows, int d, float *dst, bool centroids, cudaStream_t s);
// tf32 norm rows (B, Kpad, 8) fp32 of the fp32 centroids c (B, K, d).
int launch_prep_ext_f32(const float *c, int B, int K, int d, long long Kpad, void *cnx, cudaStream_t s);
// cnx: extension rows (B, Kpad, 16) in dtype from launch_prep_cn / finalize;
// xn: ||x||^2 per point (B, N) from launch_point_norms, or NULL (the kernel
// then computes it from its shared copy of each point tile).
// hist (nullable, zeroed by the caller, K <= 4096): the counting sort's tile
// histogram (B, ceil(N / kSortTile), K) is accumulated as the ids are written
// (run_sort_prehist then skips its histogram kernel).
int launch_assign_tc(const void *x, const void *ch, const void *cnx, const float *xn, int dtype,
                     int B, long long N, int K, int d, long long Kpad, int32_t *ids, int *err,
                     cudaStream_t s, uint32_t *hist = nullptr, unsigned long long *keys = nullptr,
                     float *xn_out = nullptr);
// keys: (B, N) zeroed scratch for the split-d variant's per-chunk work items
// (left zeroed again); NULL keeps one work item per point tile.
// xn_out (resident variant, xn NULL): the point norms computed from the shared
// tiles are also stored there, (B, N) fp32, bit-identical to launch_point_norms.
// xn[r] = ||x_r||^2 (fp32 accumulation) for `rows` rows of d 16-bit elements.
int launch_point_norms(const void *x, int dtype, long long rows, int d, float *xn, cudaStream_t s);

// counting sort: counts / offsets optional (workspace offsets are used when
// NULL); perm (sorted position -> point) and kv_out (sorted (id, point) pairs)
// are each written when not NULL.
int run_sort(Workspace *ws, const int32_t *ids, int B, long long N, int K, int32_t *counts,
             int32_t *offsets, int32_t *perm, int2 *kv_out, cudaStream_t s);
// The same single-pass sort (K <= 4096) when ws->table already holds the tile
// histogram (filled by the assign).  sort_table_bytes: its size.
bool sort_single_pass(int K);
size_t sort_table_bytes(int B, long long N, int K);
int run_sort_prehist(Workspace *ws, const int32_t *ids, int B, long long N, int K, int32_t *counts,
                     int32_t *offsets, int32_t *perm, int2 *kv_out, cudaStream_t s);

// segment reduce over the sorted (id, point) pairs kv (B, N): owner partials
// to sums (B, K, d), continuation partials to first (B, pieces_of(N), d).
int launch_segreduce(const void *x, int dtype, const int2 *kv, int B, long long N, int K, int d,
                     float *sums, float *first, cudaStream_t s);

}  // namespace fk
