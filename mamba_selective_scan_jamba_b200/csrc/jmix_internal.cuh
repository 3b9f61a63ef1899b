// Internal declarations shared by the libjmix translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "jmix.h"

namespace jmix {

constexpr int kN = 16;       // d_state (compile time)
constexpr int kConv = 4;     // d_conv (compile time)
constexpr int kMaxRank = 256;

// Error-header site of a decode row whose state slot is outside the pool.
constexpr unsigned kSiteBadSlot = 34;

// The first 256 bytes of every workspace.
struct ErrFlags {
  unsigned int timeout;    // a bounded wait ran out
  unsigned int where;      // kernel-specific code of the first wait that ran out
  unsigned int bad_input;  // device-side input check failed (cu_seqlens of a packed batch)
  unsigned int pad[61];
};
static_assert(sizeof(ErrFlags) == 256, "error header is 256 bytes");

// One mixer call (forward or decode step) after host validation.
struct Problem {
  int64_t B, L, d, R, P, T;
  float eps;
  jm_dtype io;
  const void* x;
  const void* z;
  const void* conv_w;
  const void* conv_b;
  const void* xproj_w;
  const void* dtn_w;
  const void* bn_w;
  const void* cn_w;
  const void* dtproj_w;
  const float* dt_bias;
  const float* A_log;
  const float* D;
  void* y;
  float* final_state;
  const void* init_conv;   // may be null
  const float* init_ssm;   // may be null
  void* final_conv;        // may be null; may equal init_conv
  char* ws;
  size_t ws_bytes;
  cudaStream_t stream;
  bool decode;             // jm_mixer_step
  bool zoh;                // B discretised by zero-order hold (else delta B)
  const int* cu;           // packed batch: [B + 1] token offsets (device); L == T then
  const int* sidx;         // indexed decode step: [B] state slot of each row (device), or null
  int64_t n_slots;         // indexed decode step: slots in the state pools
  const void* prepared;    // fp16 W_x and W_dt from jm_prepare_weights, or null
  int launches;            // kernels launched so far by this call
  void* const* events;     // optional per-kernel timing events (jm_set_kernel_events)
  int n_events;
  const char* names[16];   // kernel names in launch order
};

// Records events[0] (if timing events are set) before the first kernel.
void launches_begin(Problem& p);
// Counts one kernel launch (named `name` for jm_last_kernel_name) and
// records events[launches] after it.
void launched(Problem& p, const char* name);

constexpr int kMaxLaunches = 16;

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// The SIMT path of float32 io.
size_t simple_ws_bytes(const Problem& p);
cudaError_t run_simple(Problem& p);

// The bf16 path on tcgen05 tensor cores.
size_t fast_ws_bytes(const Problem& p);
// The scan schedule of the bf16 forward: time parts per sequence, two-pass or chained.
void fast_scan_schedule(int64_t B, int64_t L, int64_t d, int* n_parts, int* two_pass);
cudaError_t run_fast(Problem& p);
// Bytes of the fp16 weight copies (W_x then W_dt, each 256-byte aligned) and
// the launch that writes them.
size_t prepared_weights_bytes(int64_t d, int64_t R);
cudaError_t run_prepare_weights(int64_t d, int64_t R, const void* xproj_w, const void* dtproj_w,
                                void* out, cudaStream_t s);

// C[M, N] = A[M, K] . B[N, K]^T on tcgen05 (bf16 in, fp32 accumulation, bf16
// out, all row-major): columns [0, n_split) into C0 [M, n_split], the rest into
// C1 [M, N - n_split].  K a multiple of 8; bounded waits record into *err;
// `fold` (or null) is an earlier kernel's error header whose flags are carried
// into *err.  pdl: launched with programmatic stream serialisation.
cudaError_t gemm_bf16_tn(int64_t M, int64_t N, int64_t K, const void* A, const void* B,
                         void* C0, void* C1, int64_t n_split, ErrFlags* err,
                         const ErrFlags* fold, cudaStream_t s, bool pdl);

// Per-thread message for jm_last_error.
void set_error(const char* fmt, ...);

// Status of an error header read back to the host (JM_OK when no flag is set;
// sets the message otherwise).
jm_status status_of_flags(const ErrFlags& f);

// Launches the failure-detection self-test on `err` (cleared first): one
// thread waits, bounded, on a barrier that nothing completes, then records its
// site in *err and returns.
cudaError_t launch_wait_never(ErrFlags* err, cudaStream_t s);

}  // namespace jmix
