// jm_mixer_step_noalloc: the decode step with its scratch in a static device
// array, for callers that cannot allocate device memory themselves.
//
// Some callers have no way to get scratch memory for a step: serving engines
// that reserve all device memory up front for their caches and expose no
// allocator to plug-ins, and host code that must not touch the allocator at
// all.  This entry point needs nothing from them beyond the step's own inputs
// and outputs: its scratch is the file-scope array below, which every GPU that
// loads libjmix holds until the process exits.
#include <mutex>

#include "jmix_internal.cuh"

#define JM_API extern "C" __attribute__((visibility("default")))

namespace jmix {
namespace {

// 32 MiB: enough for a decode step of 256 sequences at Jamba v0.1 mixer shapes
// (d_inner 8192, dt_rank 256), which needs about 14 MiB.
constexpr size_t kStepScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_step_scratch[kStepScratchBytes];

std::mutex g_setup_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_step_scratch on the current device (looked up once per
// device; the array's name is only a host-side stand-in in host code).
jm_status scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    set_error("jm_mixer_step_noalloc: cudaGetDevice failed: %s", cudaGetErrorString(e));
    return JM_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    set_error("jm_mixer_step_noalloc: device %d out of range", dev);
    return JM_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_step_scratch);
    if (e != cudaSuccess || !p) {
      set_error("jm_mixer_step_noalloc: cudaGetSymbolAddress failed: %s",
                cudaGetErrorString(e));
      return JM_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return JM_OK;
}

}  // namespace
}  // namespace jmix

using namespace jmix;

JM_API jm_status jm_mixer_step_noalloc(const jm_dims* dims, const void* x_t, const void* z_t,
                                       void* conv_state, float* ssm_state, const void* conv_w,
                                       const void* conv_b, const void* xproj_w,
                                       const void* dt_norm_w, const void* b_norm_w,
                                       const void* c_norm_w, const void* dtproj_w,
                                       const float* dt_bias, const float* A_log, const float* D,
                                       void* y_t, jm_stream_t stream) {
  const size_t need = jm_mixer_step_workspace_size(dims);
  if (need == 0)  // invalid dims: let the regular entry point report why (it launches nothing)
    return jm_mixer_step(dims, x_t, z_t, conv_state, ssm_state, conv_w, conv_b, xproj_w,
                         dt_norm_w, b_norm_w, c_norm_w, dtproj_w, dt_bias, A_log, D, y_t, nullptr,
                         0, stream);
  if (need > kStepScratchBytes) {
    set_error("jm_mixer_step_noalloc: this step needs %zu bytes of scratch, more than the "
              "%zu-byte static buffer; use jm_mixer_step with a caller workspace",
              need, kStepScratchBytes);
    return JM_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  jm_status st = scratch_for_current_device(&scratch);
  if (st != JM_OK) return st;
  // The step path clears its error header itself and writes every other
  // scratch byte before reading it, so the previous call's contents never leak.
  return jm_mixer_step(dims, x_t, z_t, conv_state, ssm_state, conv_w, conv_b, xproj_w, dt_norm_w,
                       b_norm_w, c_norm_w, dtproj_w, dt_bias, A_log, D, y_t, scratch,
                       kStepScratchBytes, stream);
}

// The device-side error flags of jm_mixer_step_noalloc live in the first 256
// bytes of the static array, where a caller cannot reach them; this reads them
// back (one device-to-host copy into a host struct, no allocation).
JM_API jm_status jm_noalloc_poll_error(jm_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    set_error("CUDA error: %s", cudaGetErrorString(e));
    return JM_ERR_CUDA;
  }
  void* scratch = nullptr;
  jm_status st = scratch_for_current_device(&scratch);
  if (st != JM_OK) return st;
  ErrFlags f;
  e = cudaMemcpyAsync(&f, scratch, sizeof(f), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    set_error("CUDA error: %s", cudaGetErrorString(e));
    return JM_ERR_CUDA;
  }
  return status_of_flags(f);
}

// The failure-detection self-test aimed at the static array's error header, so
// that the report path of jm_noalloc_poll_error can be checked without a fault.
JM_API jm_status jm_noalloc_selftest_timeout(jm_stream_t stream) {
  void* scratch = nullptr;
  jm_status st = scratch_for_current_device(&scratch);
  if (st != JM_OK) return st;
  const cudaError_t e =
      launch_wait_never(static_cast<ErrFlags*>(scratch), reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    set_error("CUDA error: %s", cudaGetErrorString(e));
    return JM_ERR_CUDA;
  }
  return JM_OK;
}
