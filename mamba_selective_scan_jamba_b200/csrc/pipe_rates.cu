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
// Op codes: 0 ex2.approx.ftz.f32, 1 tanh.approx.f32, 2 rcp.approx.ftz.f32 (+1 add),
// 3 fma.rn.f32, 4 fma.rn.f32x2 (counted as 2 FMAs per lane), 5 ex2 and two
// fma.rn.f32x2 interleaved (counted as ex2 operations; checks that the two
// pipes overlap).  6 and 7 run the selective scan's 16-state recurrence alone
// (one channel per thread; per token: 16 decays exp2(delta A), the update
// h = a h + (delta u) B and the readout C . h), counted as ex2 operations:
// 6 reads each token's B and C rows from shared memory (eight 16-byte
// broadcast loads, as the scan kernel does), 7 keeps them in registers; the
// difference is the cost of those loads.
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
      if constexpr (OP == 2) v[j] = rcpf_a(v[j] + 1.0f);   // the add runs on the FMA pipe
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

// The scan recurrence alone: iters tokens of one channel per thread.  Each
// token's delta changes (so no decay is reused) and B, C come from a 32-token
// table in shared memory (kSmemBC) or from registers.
template <bool kSmemBC>
__global__ void k_recurrence(int64_t iters, float seed, float* __restrict__ sink) {
  __shared__ float4 bc[32][8];
  for (int i = threadIdx.x; i < 32 * 8; i += blockDim.x)
    bc[i / 8][i % 8] = make_float4(0.01f * (i % 7), -0.02f * (i % 5), 0.03f * (i % 3), 0.5f);
  __syncthreads();
  float2 A2[8], h[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    A2[q] = make_float2(-1.4427f * (2 * q + 1), -1.4427f * (2 * q + 2));
    h[q] = make_float2(0.f, 0.f);
  }
  float dl = 1e-3f * (1 + (threadIdx.x & 7)) * seed, u = 0.3f, ysum = 0.f;
  float4 Breg[4], Creg[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    Breg[q] = make_float4(0.1f * q, 0.2f, -0.1f, 0.05f * q);
    Creg[q] = make_float4(0.3f, -0.1f * q, 0.2f, 0.1f);
  }
  for (int64_t t = 0; t < iters; ++t) {
    const int row = (int)(t & 31);
    const float2 dl2 = make_float2(dl, dl), du2 = make_float2(dl * u, dl * u);
    float2 acc[4];
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      const float4 Bq = kSmemBC ? bc[row][q4] : Breg[q4];
      const float4 Cq = kSmemBC ? bc[row][4 + q4] : Creg[q4];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int q = q4 * 2 + half;
        const float2 Bp = half ? make_float2(Bq.z, Bq.w) : make_float2(Bq.x, Bq.y);
        const float2 Cp = half ? make_float2(Cq.z, Cq.w) : make_float2(Cq.x, Cq.y);
        const float2 x = __fmul2_rn(dl2, A2[q]);
        const float2 a = make_float2(ex2f(x.x), ex2f(x.y));
        h[q] = __ffma2_rn(a, h[q], __fmul2_rn(du2, Bp));
        acc[q4] = half ? __ffma2_rn(Cp, h[q], acc[q4]) : __fmul2_rn(Cp, h[q]);
      }
    }
    const float2 s = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
    ysum += s.x + s.y;
    dl = fmaf(dl, 0.9999f, 1e-6f);
    u = fmaf(u, -0.999f, 0.01f);
  }
  if (ysum == 12345.678f) sink[threadIdx.x] = ysum;  // keeps the work live
}

}  // namespace

// Launches op `op` on `blocks` x `threads` threads, `iters` iterations of
// kChains instructions each (ops 6, 7: iters tokens of 16 decays), on
// `stream`.  Returns 0, or a CUDA error code.
JMP_API int jmp_launch(int op, int blocks, int threads, int64_t iters, float* sink,
                       cudaStream_t stream) {
  switch (op) {
    case 0: k_pipe<0><<<blocks, threads, 0, stream>>>(iters, 0.7f, sink); break;
    case 1: k_pipe<1><<<blocks, threads, 0, stream>>>(iters, 0.2f, sink); break;
    case 2: k_pipe<2><<<blocks, threads, 0, stream>>>(iters, 1.3f, sink); break;
    case 3: k_pipe<3><<<blocks, threads, 0, stream>>>(iters, 0.5f, sink); break;
    case 4: k_pipe<4><<<blocks, threads, 0, stream>>>(iters, 0.5f, sink); break;
    case 5: k_pipe<5><<<blocks, threads, 0, stream>>>(iters, 0.7f, sink); break;
    case 6: k_recurrence<true><<<blocks, threads, 0, stream>>>(iters, 1.0f, sink); break;
    case 7: k_recurrence<false><<<blocks, threads, 0, stream>>>(iters, 1.0f, sink); break;
    default: return (int)cudaErrorInvalidValue;
  }
  return (int)cudaGetLastError();
}

// Instructions (per lane) one launch issues: blocks x threads x iters x kChains.
JMP_API int jmp_chains(void) { return kChains; }
