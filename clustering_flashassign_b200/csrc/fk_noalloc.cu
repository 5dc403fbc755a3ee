// fk_assign_noalloc: FlashAssign for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they need an
// assignment: code running under a custom or pooled allocator that owns all
// device memory, real-time loops that forbid allocation (and the implicit
// device synchronization that cudaFree can bring), or hosts that only hand
// out pre-registered buffers.  fk_assign keeps its scratch (the centroid
// norm rows the tensor-core assign reads and the kernel error word) in a per-stream workspace that it grows
// with cudaMalloc; this variant instead uses one file-scope static device
// array, so a call allocates nothing.  The caller still passes the inputs and
// the output.
//
// The array lives on every GPU that loads the library until the process
// exits.  Its size caps B * Kpad (Kpad = K rounded up to 256) at
// kNoAllocMaxRows norm rows of 32 bytes each.  Host code cannot use the array's name as a device
// address; the address is looked up once per device with
// cudaGetSymbolAddress while that device is current.
#include <mutex>

#include "fk_internal.h"

namespace fk {
namespace {

constexpr long long kNoAllocMaxRows = 1LL << 17;  // norm rows of 16 halves (4 MiB)
constexpr int kNoAllocHeader = 64;                // floats reserved for the error word

// [0, kNoAllocHeader): error word (int) and padding; then B * Kpad norm rows.
static __device__ __align__(256) float
    g_noalloc_scratch[kNoAllocHeader + kNoAllocMaxRows * kExtElems / 2];

constexpr int kMaxDevices = 64;
std::mutex g_na_mu;
float *g_na_addr[kMaxDevices] = {nullptr};

int noalloc_base(float **out) {
  int dev = 0;
  FK_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return set_error(FK_EUNSUPPORTED, "device index above 63");
  std::lock_guard<std::mutex> lk(g_na_mu);
  if (!g_na_addr[dev]) {
    void *p = nullptr;
    FK_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    g_na_addr[dev] = static_cast<float *>(p);
  }
  *out = g_na_addr[dev];
  return FK_OK;
}

}  // namespace
}  // namespace fk

using namespace fk;

extern "C" int fk_assign_noalloc(const void *x, const void *c, int B, long long N, int K, int d,
                                 int dtype, int32_t *ids, fk_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  FK_TRY(check_shape(B, N, K, d, dtype));  // the same rules as fk_assign
  if (!x || !c || !ids) return set_error(FK_EINVAL, "x, c and ids must not be NULL");
  const bool tc = dtype != FK_F32;
  if (tc && ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(c)) & 15u))
    return set_error(FK_EINVAL, "x and c must be 16-byte aligned");
  if (!tc) return launch_assign_f32((const float *)x, (const float *)c, B, N, K, d, ids, s);
  const long long Kpad = kpad_of(K);
  if ((long long)B * Kpad > kNoAllocMaxRows)
    return set_error(FK_EUNSUPPORTED, "fk_assign_noalloc: B * ceil(K/256)*256 exceeds 131072");
  float *base = nullptr;
  FK_TRY(noalloc_base(&base));
  int *err = reinterpret_cast<int *>(base);
  void *cnx = base + kNoAllocHeader;
  FK_CUDA(cudaMemsetAsync(err, 0, sizeof(int), s));  // start each call with a clear error word
  FK_TRY(launch_prep_cn(c, dtype, B, K, d, Kpad, cnx, err, s));
  return launch_assign_tc(x, c, cnx, nullptr, dtype, B, N, K, d, Kpad, ids, err, s);
}

// The error word sits in the static array, like the norm rows: read it with
// blocking copies after the stream has drained, and clear it, allocating
// nothing.
extern "C" int fk_noalloc_device_error(fk_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float *base = nullptr;
  FK_TRY(noalloc_base(&base));
  FK_CUDA(cudaStreamSynchronize(s));
  int h = DEV_OK;
  FK_CUDA(cudaMemcpy(&h, base, sizeof(int), cudaMemcpyDeviceToHost));
  if (h == DEV_OK) return FK_OK;
  const int zero = DEV_OK;
  FK_CUDA(cudaMemcpy(base, &zero, sizeof(int), cudaMemcpyHostToDevice));
  if (h == DEV_TIMEOUT) return set_error(FK_ETIMEOUT, "a kernel's bounded wait expired");
  if (h == DEV_RANGE)
    return set_error(FK_EUNSUPPORTED, "a squared norm reached 2^32, beyond the fp16 tensor-core norm digits");
  return set_error(FK_EINVAL, "unexpected device error code " + std::to_string(h));
}
