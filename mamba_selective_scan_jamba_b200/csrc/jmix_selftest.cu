// jm_selftest_timeout: proves the failure-detection path without a fault.
//
// One thread waits, through the same bounded mbarrier wait that every pipeline
// of libjmix uses, on a barrier phase that nothing completes.  The wait gives
// up after its time limit, records its site in the workspace's error header
// and returns; the host then reads JM_ERR_TIMEOUT from jm_poll_error, and the
// CUDA context stays usable.  Nothing spins without a bound and nothing traps.
#include "jmix_internal.cuh"
#include "sm100.cuh"

#define JM_API extern "C" __attribute__((visibility("default")))

namespace jmix {
namespace {

constexpr unsigned kSelftestSite = 99;

__global__ void k_wait_never(ErrFlags* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(sm100::smem_u32(&bar), 1);
    sm100::fence_mbar_init();
    // no thread arrives: phase 0 never completes, so this wait runs out
    sm100::mbar_wait(sm100::smem_u32(&bar), 0, err, kSelftestSite);
  }
}

}  // namespace

cudaError_t launch_wait_never(ErrFlags* err, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(ErrFlags), s);
  if (e != cudaSuccess) return e;
  k_wait_never<<<1, 32, 0, s>>>(err);
  return cudaGetLastError();
}

}  // namespace jmix

using namespace jmix;

JM_API jm_status jm_selftest_timeout(void* workspace, size_t ws_bytes, jm_stream_t stream) {
  if (!workspace || ws_bytes < sizeof(ErrFlags)) {
    set_error("jm_selftest_timeout: needs a workspace of at least %zu bytes", sizeof(ErrFlags));
    return JM_ERR_WORKSPACE;
  }
  const cudaError_t e = launch_wait_never(static_cast<ErrFlags*>(workspace),
                                          reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    set_error("CUDA error: %s", cudaGetErrorString(e));
    return JM_ERR_CUDA;
  }
  return JM_OK;
}
