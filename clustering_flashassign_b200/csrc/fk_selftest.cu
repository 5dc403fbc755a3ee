// fk_selftest_bounded_wait: exercises the bounded-wait path every tcgen05
// kernel of the library relies on, without any fault.  One CTA initialises an
// mbarrier that nothing ever arrives at and waits on it with the library's
// wait loop (the FlashAssign roles poll with mbarrier.test_wait and check the
// %globaltimer limit every 256 polls).  When the
// limit expires the kernel records DEV_TIMEOUT in the stream's device error
// word and returns; the host reads it as FK_ETIMEOUT and the context stays
// usable.
#include "fk_sm100.cuh"

namespace fk {
namespace {

__global__ void k_wait_selftest(unsigned long long limit_ns, int *err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = sm100::smem_u32(&bar);
  if (threadIdx.x == 0) {
    sm100::mbar_init(b, 1);
    abort_flag = 0;
    sm100::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // the same loop as mbar_wait_spin, with the caller's limit instead of 2 s
    const uint64_t t0 = sm100::globaltimer();
    for (uint32_t n = 1;; ++n) {
      if (sm100::mbar_test(b, 0)) break;  // never: nothing arrives
      if ((n & 255u) != 0) continue;
      if (abort_flag) break;
      if (sm100::globaltimer() - t0 > limit_ns) {
        abort_flag = 1;
        atomicCAS(err, DEV_OK, DEV_TIMEOUT);
        break;
      }
    }
  }
  __syncthreads();
}

}  // namespace
}  // namespace fk

using namespace fk;

extern "C" int fk_selftest_bounded_wait(long long limit_ns, fk_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (limit_ns <= 0 || limit_ns > 10000000000LL)
    return set_error(FK_EINVAL, "limit_ns must be in (0, 1e10]");
  Workspace *ws;
  FK_TRY(workspace_for(s, &ws));
  k_wait_selftest<<<1, 32, 0, s>>>((unsigned long long)limit_ns, ws->err);
  FK_TRY(launched());
  FK_CUDA(cudaGetLastError());
  return fk_device_error(stream);
}
