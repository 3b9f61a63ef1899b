// Pipe-rate microbenchmarks: the issue rates that bound the selective scan.
//
// The scan spends most of its instructions on two pipes: the multi-function
// unit (MUFU: ex2.approx for the 16 decays per token and channel, tanh.approx
// for the gate, rcp.approx) and the FMA pipe (fma.rn.f32 and the packed
// fma.rn.f32x2 of the state update).  Each kernel here keeps every SM busy with
// one of these instructions only: 8 independent dependency chains per thread,
// so the pipe, not the latency, sets the rate.  The host times a launch with
// CUDA events and divides the instruction count by it (ops/s), which becomes the
// denominator of the scan's ALU roofline.
//
// Op codes: 0 ex2.approx.ftz.f32, 1 tanh.approx.f32, 2 rcp.approx.ftz.f32,
// 3 fma.rn.f32, 4 fma.rn.f32x2 (counted as 2 FMAs per lane), 5 ex2 and two
// fma.rn.f32x2 interleaved (counted as ex2 operations; checks that the two
// pipes overlap).
#include <cuda_runtime.h>
#include <stdint.h>

#define JMP_API extern "C" __attribute__((visibility("default")))

namespace {

constexpr int kChains = 8;

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float tanhf_a(float x) {
  float y;
  asm volatile("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcpf_a(float x) {
  float y;
  asm volatile("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int OP>
__global__ void k_pipe(int64_t iters, float seed, float* __restrict__ sink) {
  float v[kChains];
  float2 w[kChains];
#pragma unroll
  for (int j = 0; j < kChains; ++j) {
    v[j] = seed + 1e-3f * (float)(threadIdx.x + j);
    w[j] = make_float2(v[j], -v[j]);
  }
  const float2 a2 = make_float2(0.999f, 1.001f), b2 = make_float2(1e-3f, -1e-3f);
  for (int64_t i = 0; i < iters; ++i) {
#pragma unroll
    for (int j = 0; j < kChains; ++j) {
      if constexpr (OP == 0) v[j] = ex2f(-v[j]);           // stays in (0.5, 1]
      if constexpr (OP == 1) v[j] = tanhf_a(v[j] + 0.5f);  // the add runs on the FMA pipe
      if constexpr (OP == 2) v[j] = rcpf_a(v[j]);
      if constexpr (OP == 3) v[j] = fmaf(v[j], 0.999f, 1e-3f);
      if constexpr (OP == 4) w[j] = __ffma2_rn(w[j], a2, b2);
      if constexpr (OP == 5) {
        v[j] = ex2f(-v[j]);
        w[j] = __ffma2_rn(w[j], a2, b2);
        w[j] = __ffma2_rn(w[j], a2, b2);
      }
    }
  }
  float acc = 0.0f;
#pragma unroll
  for (int j = 0; j < kChains; ++j) acc += v[j] + w[j].x + w[j].y;
  if (acc == 12345.678f) sink[threadIdx.x] = acc;  // keeps every chain live
}

}  // namespace

// Launches op `op` on `blocks` x `threads` threads, `iters` iterations of
// kChains instructions each, on `stream`.  Returns 0, or a CUDA error code.
JMP_API int jmp_launch(int op, int blocks, int threads, int64_t iters, float* sink,
                       cudaStream_t stream) {
  switch (op) {
    case 0: k_pipe<0><<<blocks, threads, 0, stream>>>(iters, 0.7f, sink); break;
    case 1: k_pipe<1><<<blocks, threads, 0, stream>>>(iters, 0.2f, sink); break;
    case 2: k_pipe<2><<<blocks, threads, 0, stream>>>(iters, 1.3f, sink); break;
    case 3: k_pipe<3><<<blocks, threads, 0, stream>>>(iters, 0.5f, sink); break;
    case 4: k_pipe<4><<<blocks, threads, 0, stream>>>(iters, 0.5f, sink); break;
    case 5: k_pipe<5><<<blocks, threads, 0, stream>>>(iters, 0.7f, sink); break;
    default: return (int)cudaErrorInvalidValue;
  }
  return (int)cudaGetLastError();
}

// Instructions (per lane) one launch issues: blocks x threads x iters x kChains.
JMP_API int jmp_chains(void) { return kChains; }
