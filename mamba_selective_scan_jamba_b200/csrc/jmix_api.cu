// The libjmix C ABI: host-side validation, workspace sizing and dispatch.
// Every check runs before any launch; no entry point allocates device memory.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "jmix_internal.cuh"

#define JM_API extern "C" __attribute__((visibility("default")))

namespace jmix {

static thread_local char g_msg[512];
static thread_local int g_launches = 0;
static thread_local void* const* g_events = nullptr;
static thread_local int g_n_events = 0;

void launches_begin(Problem& p) {
  if (p.events && p.n_events > 0) cudaEventRecord((cudaEvent_t)p.events[0], p.stream);
}

static thread_local const char* g_names[kMaxLaunches];

void launched(Problem& p, const char* name) {
  if (p.launches < kMaxLaunches) p.names[p.launches] = name;
  p.launches++;
  if (p.events && p.launches < p.n_events)
    cudaEventRecord((cudaEvent_t)p.events[p.launches], p.stream);
}

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
}

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return na && nb && x < y + nb && y < x + na;
}

jm_status check_dims(const jm_dims* dm, bool step) {
  if (!dm) {
    set_error("dims is NULL");
    return JM_ERR_INVALID_ARG;
  }
  if (dm->batch < 0 || dm->seqlen < 0 || dm->d_inner <= 0 || dm->dt_rank <= 0 ||
      dm->d_state <= 0 || dm->d_conv <= 0) {
    set_error("sizes must be positive (batch, seqlen >= 0)");
    return JM_ERR_INVALID_ARG;
  }
  if (step && dm->seqlen != 1) {
    set_error("jm_mixer_step needs seqlen == 1 (got %lld)", (long long)dm->seqlen);
    return JM_ERR_INVALID_ARG;
  }
  if (dm->io != JM_F32 && dm->io != JM_BF16) {
    set_error("io dtype must be JM_F32 or JM_BF16");
    return JM_ERR_INVALID_ARG;
  }
  if (dm->discretization != JM_DISC_EULER && dm->discretization != JM_DISC_ZOH) {
    set_error("discretization must be JM_DISC_EULER or JM_DISC_ZOH");
    return JM_ERR_INVALID_ARG;
  }
  if (dm->reserved != 0) {
    set_error("jm_dims.reserved must be 0");
    return JM_ERR_INVALID_ARG;
  }
  if (!(dm->eps >= 0.0f) || dm->eps != dm->eps || dm->eps > 1e30f) {
    set_error("eps must be finite and >= 0");
    return JM_ERR_INVALID_ARG;
  }
  if (dm->d_state != kN || dm->d_conv != kConv) {
    set_error("only d_state == 16 and d_conv == 4 are built (got %lld, %lld)",
              (long long)dm->d_state, (long long)dm->d_conv);
    return JM_ERR_UNSUPPORTED;
  }
  if (dm->d_inner % 8 || dm->dt_rank % 8) {
    set_error("d_inner and dt_rank must be multiples of 8 (got %lld, %lld)",
              (long long)dm->d_inner, (long long)dm->dt_rank);
    return JM_ERR_INVALID_ARG;
  }
  if (dm->dt_rank > kMaxRank) {
    set_error("dt_rank > %d is not built (got %lld)", kMaxRank, (long long)dm->dt_rank);
    return JM_ERR_UNSUPPORTED;
  }
  // element counts must stay far inside int64
  const double tok = (double)dm->batch * (double)dm->seqlen;
  if (tok * (double)dm->d_inner > 4.0e15) {
    set_error("problem too large");
    return JM_ERR_INVALID_ARG;
  }
  return JM_OK;
}

void fill_problem(Problem& p, const jm_dims* dm) {
  memset(&p, 0, sizeof(p));
  p.B = dm->batch;
  p.L = dm->seqlen;
  p.d = dm->d_inner;
  p.R = dm->dt_rank;
  p.P = dm->dt_rank + 2 * kN;
  p.T = dm->batch * dm->seqlen;
  p.eps = dm->eps;
  p.io = dm->io;
  p.zoh = dm->discretization == JM_DISC_ZOH;
}

size_t ws_bytes_for(const Problem& p) {
  return p.io == JM_BF16 ? fast_ws_bytes(p) : simple_ws_bytes(p);
}

cudaError_t dispatch(Problem& p) {
  return p.io == JM_BF16 ? run_fast(p) : run_simple(p);
}

size_t esize(jm_dtype io) { return io == JM_BF16 ? 2 : 4; }

// Pointer checks common to fwd and step.  io-dtype tensors used as TMA or
// 128-bit vector operands must be 16-byte aligned; float32 ones 16 bytes too.
jm_status check_common(const Problem& p, const char* const names[], const void* const ptrs[],
                       int n) {
  for (int i = 0; i < n; ++i) {
    if (!ptrs[i]) {
      set_error("%s is NULL", names[i]);
      return JM_ERR_INVALID_ARG;
    }
    if (!aligned(ptrs[i], 16)) {
      set_error("%s is not 16-byte aligned", names[i]);
      return JM_ERR_INVALID_ARG;
    }
  }
  return JM_OK;
}

jm_status check_ws(const Problem& p, void* ws, size_t ws_bytes) {
  size_t need = ws_bytes_for(p);
  if (!ws) {
    set_error("workspace is NULL");
    return JM_ERR_WORKSPACE;
  }
  if (!aligned(ws, 256)) {
    set_error("workspace must be 256-byte aligned");
    return JM_ERR_WORKSPACE;
  }
  if (ws_bytes < need) {
    set_error("workspace too small: %zu bytes given, %zu needed", ws_bytes, need);
    return JM_ERR_WORKSPACE;
  }
  return JM_OK;
}

}  // namespace

jm_status status_of_flags(const ErrFlags& f) {
  if (f.timeout) {
    set_error("a bounded device-side wait ran out (site %u)", f.where);
    return JM_ERR_TIMEOUT;
  }
  if (f.bad_input) {
    if (f.where == kSiteBadSlot)
      set_error("a state_idx entry is outside [0, n_slots): that row was skipped");
    else
      set_error("cu_seqlens is not 0 = c[0] <= c[1] <= ... <= c[B] = total tokens");
    return JM_ERR_INVALID_ARG;
  }
  return JM_OK;
}

namespace {

jm_status finish(Problem& p, cudaError_t e) {
  if (e != cudaSuccess) {
    set_error("CUDA error: %s", cudaGetErrorString(e));
    return JM_ERR_CUDA;
  }
  g_launches = p.launches;
  for (int i = 0; i < kMaxLaunches; ++i) g_names[i] = i < p.launches ? p.names[i] : nullptr;
  g_msg[0] = 0;
  return JM_OK;
}

}  // namespace
}  // namespace jmix

namespace jmix {
namespace {

// jm_mixer_fwd_host: at most this many sequence groups (pipeline stages).
constexpr int64_t kHostGroups = 8;

// Copy streams and events of jm_mixer_fwd_host, created once per thread (no
// device memory is allocated).
struct HostStreams {
  bool ok = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t ev_entry = nullptr, ev_exit = nullptr, ev_in[8] = {}, ev_done[8] = {};
  HostStreams() {
    const unsigned f = cudaEventDisableTiming;
    ok = cudaStreamCreateWithFlags(&in, cudaStreamNonBlocking) == cudaSuccess &&
         cudaStreamCreateWithFlags(&out, cudaStreamNonBlocking) == cudaSuccess &&
         cudaEventCreateWithFlags(&ev_entry, f) == cudaSuccess &&
         cudaEventCreateWithFlags(&ev_exit, f) == cudaSuccess;
    for (int i = 0; ok && i < 8; ++i)
      ok = cudaEventCreateWithFlags(&ev_in[i], f) == cudaSuccess &&
           cudaEventCreateWithFlags(&ev_done[i], f) == cudaSuccess;
  }
};

HostStreams& host_streams() {
  static thread_local HostStreams hs;
  return hs;
}

}  // namespace
}  // namespace jmix

using namespace jmix;

JM_API size_t jm_mixer_fwd_workspace_size(const jm_dims* dims) {
  if (check_dims(dims, false) != JM_OK) return 0;
  Problem p;
  fill_problem(p, dims);
  return ws_bytes_for(p);
}

JM_API jm_status jm_mixer_fwd_schedule(const jm_dims* dims, int* n_parts, int* two_pass) {
  if (!n_parts || !two_pass) {
    set_error("jm_mixer_fwd_schedule: NULL output pointer");
    return JM_ERR_INVALID_ARG;
  }
  jm_status st = check_dims(dims, false);
  if (st != JM_OK) return st;
  Problem p;
  fill_problem(p, dims);
  *n_parts = 1;
  *two_pass = 0;
  if (p.io == JM_BF16) fast_scan_schedule(p.B, p.L, p.d, n_parts, two_pass);
  return JM_OK;
}

JM_API size_t jm_mixer_step_workspace_size(const jm_dims* dims) {
  if (check_dims(dims, true) != JM_OK) return 0;
  Problem p;
  fill_problem(p, dims);
  p.decode = true;
  return ws_bytes_for(p);
}

static jm_status fwd_impl(const jm_dims* dims, const void* x, const void* z, const void* conv_w,
                          const void* conv_b, const void* xproj_w, const void* dt_norm_w,
                          const void* b_norm_w, const void* c_norm_w, const void* dtproj_w,
                          const float* dt_bias, const float* A_log, const float* D, void* y,
                          float* final_state, const void* init_conv_state,
                          const float* init_ssm_state, void* final_conv_state, void* workspace,
                          size_t ws_bytes, jm_stream_t stream, bool step, Problem& p,
                          const int32_t* cu = nullptr, const int32_t* sidx = nullptr,
                          int64_t n_slots = 0, const void* prepared = nullptr) {
  jm_status st = check_dims(dims, step);
  if (st != JM_OK) return st;
  fill_problem(p, dims);
  p.decode = step;
  if (cu) {  // packed batch: seqlen is the total token count
    p.T = dims->seqlen;
    p.L = dims->seqlen;
    p.cu = cu;
  }
  const char* const wn[] = {"conv_w", "conv_b", "xproj_w", "dt_norm_w", "b_norm_w", "c_norm_w",
                            "dtproj_w", "dt_bias", "A_log", "D", "final_state"};
  const void* const wp[] = {conv_w, conv_b, xproj_w, dt_norm_w, b_norm_w, c_norm_w,
                            dtproj_w, dt_bias, A_log, D, final_state};
  if ((st = check_common(p, wn, wp, 11)) != JM_OK) return st;
  const size_t es = esize(p.io);
  const size_t act = (size_t)p.T * (size_t)p.d * es;
  if (p.T > 0) {
    const char* const an[] = {"x", "z", "y"};
    const void* const ap[] = {x, z, y};
    if ((st = check_common(p, an, ap, 3)) != JM_OK) return st;
    if (overlap(y, act, x, act) || overlap(y, act, z, act)) {
      set_error("y overlaps x or z");
      return JM_ERR_INVALID_ARG;
    }
  }
  const char* const on[] = {"init_conv_state", "init_ssm_state", "final_conv_state"};
  const void* const op[] = {init_conv_state, init_ssm_state, final_conv_state};
  for (int i = 0; i < 3; ++i)
    if (op[i] && !aligned(op[i], 16)) {
      set_error("%s is not 16-byte aligned", on[i]);
      return JM_ERR_INVALID_ARG;
    }
  if ((st = check_ws(p, workspace, ws_bytes)) != JM_OK) return st;
  p.x = x;
  p.z = z;
  p.conv_w = conv_w;
  p.conv_b = conv_b;
  p.xproj_w = xproj_w;
  p.dtn_w = dt_norm_w;
  p.bn_w = b_norm_w;
  p.cn_w = c_norm_w;
  p.dtproj_w = dtproj_w;
  p.dt_bias = dt_bias;
  p.A_log = A_log;
  p.D = D;
  p.y = y;
  p.final_state = final_state;
  p.init_conv = init_conv_state;
  p.init_ssm = init_ssm_state;
  p.final_conv = final_conv_state;
  p.sidx = sidx;
  p.n_slots = n_slots;
  p.prepared = prepared;
  p.ws = static_cast<char*>(workspace);
  p.ws_bytes = ws_bytes;
  p.stream = reinterpret_cast<cudaStream_t>(stream);
  p.launches = 0;
  p.events = g_events;
  p.n_events = g_n_events;
  if (p.B == 0) return finish(p, cudaSuccess);
  if (p.T == 0) {
    // nothing to scan: the final states are the initial ones
    const size_t ssz = (size_t)p.B * p.d * kN * 4, csz = (size_t)p.B * p.d * (kConv - 1) * es;
    cudaError_t e = init_ssm_state
                        ? cudaMemcpyAsync(final_state, init_ssm_state, ssz,
                                          cudaMemcpyDeviceToDevice, p.stream)
                        : cudaMemsetAsync(final_state, 0, ssz, p.stream);
    if (e == cudaSuccess && final_conv_state && final_conv_state != init_conv_state)
      e = init_conv_state ? cudaMemcpyAsync(final_conv_state, init_conv_state, csz,
                                            cudaMemcpyDeviceToDevice, p.stream)
                          : cudaMemsetAsync(final_conv_state, 0, csz, p.stream);
    return finish(p, e);
  }
  return finish(p, dispatch(p));
}

JM_API jm_status jm_mixer_fwd(const jm_dims* dims, const void* x, const void* z,
                              const void* conv_w, const void* conv_b, const void* xproj_w,
                              const void* dt_norm_w, const void* b_norm_w, const void* c_norm_w,
                              const void* dtproj_w, const float* dt_bias, const float* A_log,
                              const float* D, void* y, float* final_state,
                              const void* init_conv_state, const float* init_ssm_state,
                              void* final_conv_state, void* workspace, size_t ws_bytes,
                              jm_stream_t stream) {
  Problem p;
  return fwd_impl(dims, x, z, conv_w, conv_b, xproj_w, dt_norm_w, b_norm_w, c_norm_w, dtproj_w,
                  dt_bias, A_log, D, y, final_state, init_conv_state, init_ssm_state,
                  final_conv_state, workspace, ws_bytes, stream, false, p);
}

JM_API size_t jm_mixer_fwd_varlen_workspace_size(const jm_dims* dims) {
  // the packed batch needs what a batch of one sequence of T tokens needs, plus
  // nothing per sequence beyond the states the caller passes
  if (check_dims(dims, false) != JM_OK || dims->io != JM_BF16) return 0;
  Problem p;
  fill_problem(p, dims);
  p.T = dims->seqlen;
  p.L = dims->seqlen;
  p.cu = reinterpret_cast<const int*>(uintptr_t(1));  // layout of the packed form
  return ws_bytes_for(p);
}

JM_API jm_status jm_mixer_fwd_varlen(const jm_dims* dims, const int32_t* cu_seqlens,
                                     const void* x, const void* z, const void* conv_w,
                                     const void* conv_b, const void* xproj_w,
                                     const void* dt_norm_w, const void* b_norm_w,
                                     const void* c_norm_w, const void* dtproj_w,
                                     const float* dt_bias, const float* A_log, const float* D,
                                     void* y, float* final_state, const void* init_conv_state,
                                     const float* init_ssm_state, void* final_conv_state,
                                     void* workspace, size_t ws_bytes, jm_stream_t stream) {
  jm_status st = check_dims(dims, false);
  if (st != JM_OK) return st;
  if (dims->io != JM_BF16) {
    set_error("jm_mixer_fwd_varlen is built for bf16 io only");
    return JM_ERR_UNSUPPORTED;
  }
  if (!cu_seqlens) {
    set_error("cu_seqlens is NULL");
    return JM_ERR_INVALID_ARG;
  }
  if (!aligned(cu_seqlens, 4)) {
    set_error("cu_seqlens is not 4-byte aligned");
    return JM_ERR_INVALID_ARG;
  }
  if (dims->seqlen > 0x7fffffffLL) {
    set_error("total tokens must fit int32 offsets");
    return JM_ERR_INVALID_ARG;
  }
  Problem p;
  return fwd_impl(dims, x, z, conv_w, conv_b, xproj_w, dt_norm_w, b_norm_w, c_norm_w, dtproj_w,
                  dt_bias, A_log, D, y, final_state, init_conv_state, init_ssm_state,
                  final_conv_state, workspace, ws_bytes, stream, false, p, cu_seqlens);
}

JM_API jm_status jm_mixer_step(const jm_dims* dims, const void* x_t, const void* z_t,
                               void* conv_state, float* ssm_state, const void* conv_w,
                               const void* conv_b, const void* xproj_w, const void* dt_norm_w,
                               const void* b_norm_w, const void* c_norm_w, const void* dtproj_w,
                               const float* dt_bias, const float* A_log, const float* D,
                               void* y_t, void* workspace, size_t ws_bytes, jm_stream_t stream) {
  if (!conv_state || !ssm_state) {
    set_error("conv_state and ssm_state are required");
    return JM_ERR_INVALID_ARG;
  }
  Problem p;
  return fwd_impl(dims, x_t, z_t, conv_w, conv_b, xproj_w, dt_norm_w, b_norm_w, c_norm_w,
                  dtproj_w, dt_bias, A_log, D, y_t, ssm_state, conv_state, ssm_state, conv_state,
                  workspace, ws_bytes, stream, true, p);
}

JM_API size_t jm_prepared_weights_size(const jm_dims* dims) {
  if (check_dims(dims, false) != JM_OK || dims->io != JM_BF16) return 0;
  return prepared_weights_bytes(dims->d_inner, dims->dt_rank);
}

JM_API jm_status jm_prepare_weights(const jm_dims* dims, const void* xproj_w,
                                    const void* dtproj_w, void* prepared, size_t bytes,
                                    jm_stream_t stream) {
  jm_status st = check_dims(dims, false);
  if (st != JM_OK) return st;
  if (dims->io != JM_BF16) {
    set_error("jm_prepare_weights: only bf16 weights are converted (float32 io uses them as is)");
    return JM_ERR_UNSUPPORTED;
  }
  if (!xproj_w || !dtproj_w || !prepared) {
    set_error("jm_prepare_weights: NULL pointer");
    return JM_ERR_INVALID_ARG;
  }
  if (!aligned(xproj_w, 16) || !aligned(dtproj_w, 16) || !aligned(prepared, 256)) {
    set_error("jm_prepare_weights: weights must be 16-byte aligned, prepared 256-byte aligned");
    return JM_ERR_INVALID_ARG;
  }
  const size_t need = prepared_weights_bytes(dims->d_inner, dims->dt_rank);
  if (bytes < need) {
    set_error("jm_prepare_weights: %zu bytes given, %zu needed", bytes, need);
    return JM_ERR_WORKSPACE;
  }
  const cudaError_t e = run_prepare_weights(dims->d_inner, dims->dt_rank, xproj_w, dtproj_w,
                                            prepared, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    set_error("CUDA error: %s", cudaGetErrorString(e));
    return JM_ERR_CUDA;
  }
  return JM_OK;
}

JM_API jm_status jm_mixer_step_indexed(const jm_dims* dims, const int32_t* state_idx,
                                       int64_t n_slots, const void* x_t, const void* z_t,
                                       void* conv_pool, float* ssm_pool, const void* conv_w,
                                       const void* conv_b, const void* xproj_w,
                                       const void* dt_norm_w, const void* b_norm_w,
                                       const void* c_norm_w, const void* dtproj_w,
                                       const float* dt_bias, const float* A_log, const float* D,
                                       const void* prepared, void* y_t, void* workspace,
                                       size_t ws_bytes, jm_stream_t stream) {
  jm_status st = check_dims(dims, true);
  if (st != JM_OK) return st;
  if (dims->io != JM_BF16) {
    set_error("jm_mixer_step_indexed is built for bf16 io only");
    return JM_ERR_UNSUPPORTED;
  }
  if (!conv_pool || !ssm_pool) {
    set_error("conv_pool and ssm_pool are required");
    return JM_ERR_INVALID_ARG;
  }
  if (dims->batch > 0 && (!state_idx || !aligned(state_idx, 4))) {
    set_error("state_idx must be a 4-byte aligned device array of batch entries");
    return JM_ERR_INVALID_ARG;
  }
  if (n_slots < dims->batch || n_slots > 0x7fffffffLL || (dims->batch > 0 && n_slots < 1)) {
    set_error("n_slots must be in [batch, 2^31) (the batch's slots are distinct), got %lld",
              (long long)n_slots);
    return JM_ERR_INVALID_ARG;
  }
  if (prepared && !aligned(prepared, 256)) {
    set_error("prepared weights must be 256-byte aligned");
    return JM_ERR_INVALID_ARG;
  }
  Problem p;
  return fwd_impl(dims, x_t, z_t, conv_w, conv_b, xproj_w, dt_norm_w, b_norm_w, c_norm_w,
                  dtproj_w, dt_bias, A_log, D, y_t, ssm_pool, conv_pool, ssm_pool, conv_pool,
                  workspace, ws_bytes, stream, true, p, nullptr, state_idx, n_slots, prepared);
}

JM_API jm_status jm_mixer_fwd_host(const jm_dims* dims, const void* x_host, const void* z_host,
                                   void* y_host, float* final_state_host, void* x_dev,
                                   void* z_dev, void* y_dev, float* final_state_dev,
                                   const void* conv_w, const void* conv_b, const void* xproj_w,
                                   const void* dt_norm_w, const void* b_norm_w,
                                   const void* c_norm_w, const void* dtproj_w,
                                   const float* dt_bias, const float* A_log, const float* D,
                                   void* workspace, size_t ws_bytes, jm_stream_t stream) {
  jm_status st = check_dims(dims, false);
  if (st != JM_OK) return st;
  const size_t act = (size_t)dims->batch * dims->seqlen * dims->d_inner * esize(dims->io);
  if (act && (!x_host || !z_host || !y_host)) {
    set_error("host buffers are required");
    return JM_ERR_INVALID_ARG;
  }
  if (!final_state_host) {
    set_error("final_state_host is NULL");
    return JM_ERR_INVALID_ARG;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // validate everything before the first copy is queued
  Problem probe;
  fill_problem(probe, dims);
  if ((st = check_ws(probe, workspace, ws_bytes)) != JM_OK) return st;
  if (act && (!x_dev || !z_dev || !y_dev)) {
    set_error("device staging buffers are required");
    return JM_ERR_INVALID_ARG;
  }
  // The batch runs in groups of whole sequences so that copies overlap compute:
  // group g's inputs go up on an inbound stream, its forward runs on `stream`
  // once they have landed, and its outputs come down on an outbound stream
  // while later groups compute (PCIe moves both directions at once).  Each group
  // is independent sequences, and the groups reuse the workspace in stream
  // order; if a group would need more workspace than given, one group is used.
  const int64_t B = dims->batch, L = dims->seqlen, d = dims->d_inner;
  const size_t es = esize(dims->io);
  int64_t groups = B >= 2 ? (B < kHostGroups ? B : kHostGroups) : 1;
  int64_t bg = groups > 0 ? (B + groups - 1) / groups : 0;
  if (groups > 1) {
    jm_dims gd = *dims;
    gd.batch = bg;
    if (jm_mixer_fwd_workspace_size(&gd) > ws_bytes) {
      groups = 1;
      bg = B;
    } else {
      groups = (B + bg - 1) / bg;
    }
  }
  HostStreams& hs = host_streams();
  if (!hs.ok) {
    set_error("could not create the copy streams");
    return JM_ERR_CUDA;
  }
  cudaError_t e = cudaEventRecord(hs.ev_entry, s);  // earlier work on `stream` comes first
  if (e == cudaSuccess) e = cudaStreamWaitEvent(hs.in, hs.ev_entry, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(hs.out, hs.ev_entry, 0);
  int launches = 0;
  for (int64_t g = 0; g < groups && e == cudaSuccess; ++g) {
    const int64_t b0 = g * bg, nb = (B - b0) < bg ? (B - b0) : bg;
    const size_t a0 = (size_t)b0 * L * d * es, an = (size_t)nb * L * d * es;
    const size_t s0 = (size_t)b0 * d * kN * 4, sn = (size_t)nb * d * kN * 4;
    char* xd = static_cast<char*>(x_dev) + a0;
    char* zd = static_cast<char*>(z_dev) + a0;
    char* yd = static_cast<char*>(y_dev) + a0;
    if (an) {
      e = cudaMemcpyAsync(xd, static_cast<const char*>(x_host) + a0, an, cudaMemcpyHostToDevice,
                          hs.in);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(zd, static_cast<const char*>(z_host) + a0, an,
                            cudaMemcpyHostToDevice, hs.in);
    }
    if (e == cudaSuccess) e = cudaEventRecord(hs.ev_in[g], hs.in);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, hs.ev_in[g], 0);
    if (e != cudaSuccess) break;
    jm_dims gd = *dims;
    gd.batch = nb;
    Problem p;
    st = fwd_impl(&gd, xd, zd, conv_w, conv_b, xproj_w, dt_norm_w, b_norm_w, c_norm_w, dtproj_w,
                  dt_bias, A_log, D, yd, final_state_dev + s0 / 4, nullptr, nullptr, nullptr,
                  workspace, ws_bytes, stream, false, p);
    if (st != JM_OK) return st;
    launches += p.launches;
    e = cudaEventRecord(hs.ev_done[g], s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(hs.out, hs.ev_done[g], 0);
    if (e == cudaSuccess && an)
      e = cudaMemcpyAsync(static_cast<char*>(y_host) + a0, yd, an, cudaMemcpyDeviceToHost, hs.out);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(reinterpret_cast<char*>(final_state_host) + s0,
                          reinterpret_cast<char*>(final_state_dev) + s0, sn,
                          cudaMemcpyDeviceToHost, hs.out);
  }
  // the caller's stream covers every copy from here on
  if (e == cudaSuccess) e = cudaEventRecord(hs.ev_exit, hs.out);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, hs.ev_exit, 0);
  if (e != cudaSuccess) {
    set_error("CUDA error: %s", cudaGetErrorString(e));
    return JM_ERR_CUDA;
  }
  g_launches = launches;
  return JM_OK;
}

JM_API jm_status jm_poll_error(void* workspace, jm_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    set_error("CUDA error: %s", cudaGetErrorString(e));
    return JM_ERR_CUDA;
  }
  if (!workspace) {
    set_error("workspace is NULL");
    return JM_ERR_INVALID_ARG;
  }
  ErrFlags f;
  e = cudaMemcpyAsync(&f, workspace, sizeof(f), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    set_error("CUDA error: %s", cudaGetErrorString(e));
    return JM_ERR_CUDA;
  }
  return status_of_flags(f);
}

JM_API const char* jm_last_error(void) { return g_msg; }

JM_API int jm_last_launch_count(void) { return g_launches; }

JM_API const char* jm_last_kernel_name(int index) {
  if (index < 0 || index >= kMaxLaunches || index >= g_launches || !g_names[index]) return "";
  return g_names[index];
}

JM_API jm_status jm_set_kernel_events(void* const* events, int n_events) {
  if (n_events < 0 || (n_events > 0 && !events)) {
    set_error("events must be NULL with n_events == 0, or an array of n_events events");
    return JM_ERR_INVALID_ARG;
  }
  g_events = n_events ? events : nullptr;
  g_n_events = n_events;
  return JM_OK;
}
